// fwd_softmax.cuh -- softmax warpgroups of the prefill kernel.
//
// Thread r of warpgroup X owns query row r of head slot X (TMEM lane r).  Per
// key tile: read S from TMEM and release the S buffer at once (the next
// QK^T overlaps the exponentials); classify each 32-key chunk for this warp
// as hidden (skipped: its P is zero), partly visible (masked per element) or
// fully visible; online softmax in log2 units with a running base m and sum
// l; P in fp16 into TMEM, one half at a time.
//
// P is fp16, not bf16: its 11-bit significand keeps the P V product's
// rounding about eight times smaller, which the output needs -- a bf16
// output of magnitude 2..4 already spends up to 7.8e-3 of the 1e-2 bar on its
// own rounding.
//
// The base.  A row's first visible tile sets m to its maximum, so that tile's
// largest P is exactly 1 (and the row sum stays >= 1 from then on); while the
// row has seen fewer than 64 keys it also takes later tiles' maxima.  After
// that, tiles reuse m as it stands and skip the row maximum: any base gives the
// same O / l, and fp16 P (down to its subnormals, far below 1 / l) and fp32
// sums keep their precision at any scale the range allows.  The only risk
// is range: fp16 ends at 65504, so the tile's sum is checked afterwards --
// above 2^15 (or not finite) the warp recomputes the tile against its true
// maximum (the scores are still in registers) and rescales l and O.  In
// attention the scores after the first tile rarely exceed its maximum by 8
// (log2 units) over a whole row, so the redo path is cold; a row whose first
// tile is fully masked keeps m = -inf and takes the maximum path again on
// the next one.
//
// Epilogue: the sink joins the max and the sum once -- M = max(m, sink),
// l' = l 2^(m-M) + 2^(sink-M) (no term for sink = -inf) -- then
// O 2^(m-M) / l' in bf16 and LSE = (M + log2 l') ln 2.  A unit's epilogue
// runs inside the next unit's first tile (PendingRow below).
#pragma once

#include "fwd_common.cuh"

namespace gptoss {

// P enters P V as fp16 (largest finite value 65504): a tile whose row sum
// stays at or below 2^15 has every element at or below 2^15.
constexpr float kMaxTileSum = 32768.0f;  // 2^15

// Row maximum of the raw scores over the chunks this warp can see (masked
// elements already hold -inf); -inf when none is visible.
__device__ __forceinline__ float tile_max(const uint32_t (&sr)[4][32], const int (&cls)[4]) {
  float mc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    mc[c] = -INFINITY;
    if (cls[c] != 0) {
#pragma unroll
      for (int e = 0; e < 32; e += 2) mc[c] = fmax3(mc[c], __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
    }
  }
  return fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
}

// Reads this warp's 32 rows x 128 scores of S from TMEM and sets the hidden
// elements of partly visible chunks to -inf (row qi, at key index gi =
// qi + delta, sees keys [gi - window + 1, min(gi, Lk - 1)]; k0 is the tile's
// first key).  kWindow = false: no window, only the causal bound.
template <bool kWindow>
__device__ __forceinline__ void load_masked_s(uint32_t taddr, const int (&cls)[4], int gi, int k0, int Lk,
                                              int window, uint32_t (&sr)[4][32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32(taddr + c * 32, sr[c]);
  tmem_wait_ld();
  const int c_hi = min(gi, Lk - 1) - k0;  // visible columns of this row: [c_lo, c_hi]
  const int c_lo = kWindow ? gi - window + 1 - k0 : -1;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (cls[c] == 1) {  // warp-uniform branch
      const int lo_c = c_lo - 32 * c, hi_c = c_hi - 32 * c;
      if (kWindow) {
        // this row's visible columns of the chunk, [lo_c, hi_c], as a bit
        // mask: one bit test and select per element (measured: 9 % faster on
        // the sliding window than comparing each column with both bounds)
        const uint32_t upto = hi_c >= 31 ? 0xffffffffu : (hi_c < 0 ? 0u : (2u << hi_c) - 1u);
        const uint32_t from = lo_c <= 0 ? 0xffffffffu : (lo_c > 31 ? 0u : ~((1u << lo_c) - 1u));
        const uint32_t vis = upto & from;
#pragma unroll
        for (int e = 0; e < 32; ++e) sr[c][e] = (vis & (1u << e)) ? sr[c][e] : __float_as_uint(-INFINITY);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e > hi_c) sr[c][e] = __float_as_uint(-INFINITY);
      }
    }
  }
}

// P = 2^(s sl - base) for chunks (2 half, 2 half + 1) as 32 packed bf16 pairs;
// adds the fp32 values to (rs0, rs1).  Hidden chunks give zeros.
__device__ __forceinline__ void exp_half(const uint32_t (&sr)[4][32], const int (&cls)[4], int half, float sl,
                                         float nb, float& rs0, float& rs1, uint32_t (&pk)[32]) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * half + cc;
    if (cls[c] == 0) {
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[cc * 16 + e] = 0u;
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = fmaf(__uint_as_float(sr[c][2 * e]), sl, nb);
        const float x1 = fmaf(__uint_as_float(sr[c][2 * e + 1]), sl, nb);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        rs0 += p0;
        rs1 += p1;
        pk[cc * 16 + e] = pack_f16(p0, p1);
      }
    }
  }
}

// A finished row awaiting its epilogue: the epilogue of a unit runs during
// the next unit's first tile, right after that tile's wait for the previous
// P V product -- which is this unit's last -- so the product's latency hides
// behind the next unit's S read and first exponentials instead of stalling
// the warp at the end of every unit.
struct PendingRow {
  float m, l, sink;
  int64_t out_row;  // element offset of the output row (head included); -1: nothing to store
  int64_t lse_idx;  // -1: no lse
};
// (out_row indexes p.out with its strides, or the dense fp32 p.out_f32.)

// O / l with the sink folded once (M = max(m, sink), l' = l 2^(m - M) +
// 2^(sink - M)), in bf16, and LSE = (M + log2 l') ln 2.  O (kD columns) must
// be complete.
template <int kD>
__device__ __forceinline__ void fwd_epilogue_row(const FwdParams& p, uint32_t o_addr, const PendingRow& pr) {
  const float M = fmaxf(pr.m, pr.sink);
  const float a = pr.m == -INFINITY ? 0.f : ex2_approx(pr.m - M);
  const float l_fin = pr.l * a + (pr.sink == -INFINITY ? 0.f : ex2_approx(pr.sink - M));
  const float inv = a / l_fin;
#pragma unroll
  for (int c = 0; c < kD / 32; ++c) {
    uint32_t ov[32];
    tmem_ld32(o_addr + c * 32, ov);
    tmem_wait_ld();
    if (pr.out_row >= 0 && p.out_f32 != nullptr) {
      float* dst = p.out_f32 + pr.out_row + c * 32;
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        float4 v;
        v.x = __uint_as_float(ov[4 * c4 + 0]) * inv;
        v.y = __uint_as_float(ov[4 * c4 + 1]) * inv;
        v.z = __uint_as_float(ov[4 * c4 + 2]) * inv;
        v.w = __uint_as_float(ov[4 * c4 + 3]) * inv;
        *reinterpret_cast<float4*>(dst + 4 * c4) = v;
      }
    } else if (pr.out_row >= 0) {
      __nv_bfloat16* dst = p.out + pr.out_row + c * 32;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint4 v;
        const int e = c8 * 8;
        v.x = pack_bf16(__uint_as_float(ov[e + 0]) * inv, __uint_as_float(ov[e + 1]) * inv);
        v.y = pack_bf16(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
        v.z = pack_bf16(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
        v.w = pack_bf16(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
        *reinterpret_cast<uint4*>(dst + c8 * 8) = v;
      }
    }
  }
  if (pr.out_row >= 0 && pr.lse_idx >= 0) p.lse[pr.lse_idx] = (M + log2f(l_fin)) * kLn2;
}

// kWindow: the call has a sliding window (window > 0); false compiles the
// causal-only masks (a smaller loop for the full-context layers).  kD: head
// size, the width of O (64: two head slots per CTA, O_X at 384 + 64 X; 128:
// one slot, O at 384 .. 511).  Smem: the kernel's shared-memory layout (its
// s_full per slot and S buffer, p_full per S buffer, o_done per slot).
template <bool kWindow, int kD = kHeadDim, typename Smem = FwdSmem>
__device__ __forceinline__ void fwd_softmax_role(const FwdParams& p, Smem& sm, uint32_t tmem, int X) {
  const int window = kWindow ? p.window : 0;
  const int wq = (threadIdx.x >> 5) & 3;  // warp within the warpgroup = TMEM lane quarter
  const int r = threadIdx.x & 127;        // query row of the tile
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  constexpr uint32_t kSlots = kD == kHeadDim ? 2 : 1;  // head slots per CTA
  // the tensor-memory layout (fwd_common.cuh): three S buffers, or per slot
  // for the sliding-window kernel at D = 64
  constexpr bool kTri = !(kWindow && kD == kHeadDim);
  const uint32_t colO = kTri ? kColO + (kD == kHeadDim ? X * 64 : 0) : X * 256 + 192;
  const bool thd = p.cu_seqlens != nullptr;
  const float sl = p.scale_log2;
  uint32_t t = 0;  // running tile count of this CTA
  bool pending = false;
  PendingRow pr;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit w;
    if (!make_unit<kD == kHeadDim>(p, u, w)) continue;
    const int h = X == 0 ? w.h0 : w.h1;
    const int qi = w.q0 + r;
    // rows of this warp, as key indices (query row i sits at key index i + delta)
    const int qw_lo = w.q0 + wq * 32 + p.delta, qw_hi = qw_lo + 31;
    const float sink = p.sinks != nullptr ? __ldg(p.sinks + h) * kLog2e : -INFINITY;
    float m_run = -INFINITY;
    float l_run = 0.f;
    int n_seen = 0;  // visible keys this row's base has seen so far
    for (int j = 0; j < w.n_kt; ++j, ++t) {
      const int k0 = (w.j_lo + j) * kFwdTile;
      // three-buffer layout: score product t * slots + X sits in S buffer
      // (t * slots + X) mod 3 and P goes over it; this is the slot's use t / 3
      // of that buffer (each slot takes every buffer once in three tiles).
      // Per-slot layout: S_X, then P_X beside it; b = X indexes p_full.
      const uint32_t b = kTri ? (t * kSlots + X) % kSBufs : X;
      const uint32_t colS = kTri ? b * 128 : X * 256, colP = kTri ? colS : colS + 128;
      if (!mbar_wait_warp(&sm.s_full[X][kTri ? b : 0], (kTri ? t / kSBufs : t) & 1, p.wait_ns)) return;
      tc_fence_after();
      // chunk classes for this warp: 0 hidden, 1 partly visible, 2 visible
      int cls[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int kl = k0 + 32 * c, kh = kl + 31;
        const bool hidden = kl > min(qw_hi, w.Lk - 1) || (window > 0 && kh < qw_lo - window + 1);
        const bool full = kh <= qw_lo && kh <= w.Lk - 1 && (window == 0 || kl >= qw_hi - window + 1);
        cls[c] = hidden ? 0 : (full ? 2 : 1);
      }
      uint32_t sr[4][32];
      load_masked_s<kWindow>(lane_base + colS, cls, qi + p.delta, k0, w.Lk, window, sr);
      if (!kTri) {  // per slot: the next S may go into S_X now
        tc_fence_before();
        mbar_arrive(&sm.s_free[X]);
      }
      float alpha = 1.f;
      bool rescale = false;
      // A row whose base rests on few keys (none yet, or fewer than 64) takes
      // this tile's maximum -- the whole warp does, so the branch stays
      // uniform.  With the maximum known, every P of the tile is at most
      // 2^(max - base), so the base moves (the lazy O rescale) only when that
      // would leave the fp16 range, and the tile needs no range check after
      // its exponentials.  In the sliding window every unit starts with rows
      // that see a handful of keys in their first tile; moving their base at
      // every larger maximum, or redoing tiles whose sum passes 2^15, cost a
      // quarter of the kernel.  Once a row has seen 64 keys its base stands
      // and later tiles skip the maximum.
      const int gi = qi + p.delta;  // this row's visible keys in the tile: [v_lo, v_hi]
      const int v_hi = min(min(gi, w.Lk - 1), k0 + kFwdTile - 1);
      const int v_lo = max(k0, window > 0 ? gi - window + 1 : k0);
      const bool young = n_seen < 64;
      n_seen += max(0, v_hi - v_lo + 1);
      // One copy of the maximum and of the exponentials, in a rolled loop of at
      // most two passes: the hot loop must fit the instruction cache (with a
      // second, unrolled copy for the cold redo the warps stalled on
      // instruction fetch).  A pass that takes the maximum needs no range
      // check; a pass that fails the check takes the maximum and runs again
      // only if some row's base moved.
      bool max_pass = __any_sync(0xffffffffu, young);
      // per slot: P(t) overwrites P(t-1), so the previous P V must have
      // completed before the first store
      bool waited = kTri || t == 0;
      float rs = 0.f;
      for (int pass = 0;; ++pass) {
        if (max_pass) {
          const float m_cand = tile_max(sr, cls) * sl;
          const bool moved = m_cand > m_run + kRescaleThreshold;
          if (moved) {
            alpha *= ex2_approx(m_run - m_cand);  // 0 when m_run is -inf
            m_run = m_cand;
            rescale = true;
          }
          if (pass > 0 && !__any_sync(0xffffffffu, moved)) break;  // the first pass's P stand
        }
        const float nb = m_run == -INFINITY ? 0.f : -m_run;
        float rs0 = 0.f, rs1 = 0.f;
        uint32_t pk[32];
        exp_half(sr, cls, 0, sl, nb, rs0, rs1, pk);
        if (!waited) {
          if (!mbar_wait_warp(&sm.o_done[X], (t - 1) & 1, p.wait_ns)) return;
          tc_fence_after();
          waited = true;
        }
        // three-buffer layout: over the S columns this thread has already
        // read (its own lane); the buffer's previous P was consumed before
        // this S was computed
        tmem_st32(lane_base + colP, pk);
        exp_half(sr, cls, 1, sl, nb, rs0, rs1, pk);
        tmem_st32(lane_base + colP + 32, pk);
        rs = rs0 + rs1;
        if (max_pass || !__any_sync(0xffffffffu, !(rs <= kMaxTileSum))) break;
        max_pass = true;
      }
      // The previous tile's P V, waited for once per tile after this tile's P
      // is stored (by then it has usually completed): every poll of o_done
      // then follows the one of the phase before, so the parity test cannot
      // mistake a phase two ahead for a completed one, and O holds every
      // product up to this tile's.
      if (kTri && t > 0) {
        if (!mbar_wait_warp(&sm.o_done[X], (t - 1) & 1, p.wait_ns)) return;
        tc_fence_after();
      }
      // the previous unit's rows (its last P V has completed); this unit's
      // first P V, which restarts O, waits for p_full below
      if (j == 0 && pending) {
        fwd_epilogue_row<kD>(p, lane_base + colO, pr);
        pending = false;
      }
      // warp-collective TMEM access: the whole warp rescales O when any row
      // needs it (alpha is 1 for the rows that do not)
      if (__any_sync(0xffffffffu, rescale && j > 0)) {
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(lane_base + colO + c * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(lane_base + colO + c * 32, ov);
        }
      }
      l_run = l_run * alpha + rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[b]);
    }
    // this unit's epilogue waits for the next unit's first tile (or the end)
    pr.m = m_run;
    pr.l = l_run;
    pr.sink = sink;
    pr.out_row = -1;
    pr.lse_idx = -1;
    // the row's logical coordinates (token, head) lie inside the call's tensors
    if (qi < w.L && !(X == 1 && w.dup) &&
        index_ok(h < p.Hq && (thd ? w.seq_start + qi < p.T : (w.b < p.B && qi < p.S)))) {
      pr.out_row = p.out_f32 != nullptr
                       ? ((static_cast<int64_t>(w.b) * p.S + qi) * p.Hq + h) * kD
                       : (thd ? static_cast<int64_t>(w.seq_start + qi) * p.so.tok
                              : static_cast<int64_t>(w.b) * p.so.batch + static_cast<int64_t>(qi) * p.so.tok) +
                             static_cast<int64_t>(h) * p.so.head;
      if (p.lse != nullptr)
        pr.lse_idx = thd ? static_cast<int64_t>(h) * p.T + w.seq_start + qi
                         : (static_cast<int64_t>(w.b) * p.Hq + h) * p.S + qi;
    }
    pending = true;
  }
  if (pending) {  // the last unit: wait for its last P V product
    if (!mbar_wait_warp(&sm.o_done[X], (t - 1) & 1, p.wait_ns)) return;
    tc_fence_after();
    fwd_epilogue_row<kD>(p, lane_base + colO, pr);
  }
  tc_fence_before();
}

}  // namespace gptoss
