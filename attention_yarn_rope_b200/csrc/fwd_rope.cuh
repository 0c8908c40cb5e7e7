// fwd_rope.cuh -- rope warpgroup of the prefill kernel: RoPE fused into the
// Q and K tile loads (NeMo AutoModel gpt_oss.rope_utils page,
// apply_rotary_emb_qk: half-split pairs, concentration applied).
//
// TMA lands raw bf16 Q and K tiles (128 rows x 64 features, 128B-swizzled) in
// shared memory; this warpgroup rotates them in place and leaves fp16 values
// for the QK^T product.  Thread (w, l) owns pairs (2pb, 2pb+32) and
// (2pb+1, 2pb+33), pb = l % 16, of rows ro, ro+8, ..., ro+120 with
// ro = w + 4 (l / 16): the two half-warps touch rows 4 apart, whose swizzled
// chunks fall in disjoint banks.  The angle of row ro + 8k is the row-ro seed
// times (cos 8f, sin 8f)^k: one double-precision seed per tile and pair
// (rope_cs), the rest complex multiplications, so no transcendental per
// element.  With explicit positions every row gets its own seed.
#pragma once

#include "fwd_common.cuh"

namespace gptoss {

struct RopeLane {
  int ro;                 // first row of this thread
  uint32_t w_lo, w_hi;    // byte offsets of its two words in row ro
  double f0, f1;          // inverse frequencies of its two pairs
  float2 step0, step1;    // (cos 8f, sin 8f)
};

// Rotates the 16 rows this thread owns; rows at or past n_valid (beyond the
// sequence) are left as they are -- their scores are masked.  (c0, c1) is
// the angle of row ro for the thread's two pairs, concentration included;
// row ro + 8k gets (c, s) * (cos 8f, sin 8f)^k.  Explicit positions give
// every row its own double-precision seed.  (Measured: rotating row by row
// in a 4-way unrolled loop beats loading all 32 words up front.)
__device__ __forceinline__ void rotate_tile(const FwdParams& p, const RopeLane& rl, uint8_t* tile, float2 c0,
                                            float2 c1, int n_valid, const int32_t* pos_row0) {
  const bool explicit_pos = pos_row0 != nullptr;
#pragma unroll 4
  for (int kk = 0; kk < 16; ++kk) {
    const int r = rl.ro + 8 * kk;
    if (r < n_valid) {
      if (explicit_pos) {
        const int pos = __ldg(pos_row0 + r);
        c0 = rope_cs(pos, rl.f0, p.tab.conc);
        c1 = rope_cs(pos, rl.f1, p.tab.conc);
      }
      uint32_t* plo = reinterpret_cast<uint32_t*>(tile + rl.w_lo + kk * 1024);
      uint32_t* phi = reinterpret_cast<uint32_t*>(tile + rl.w_hi + kk * 1024);
      uint32_t lo = *plo, hi = *phi;
      rotate_words(lo, hi, c0, c1);
      *plo = lo;
      *phi = hi;
    }
    if (!explicit_pos) {
      c0 = cmul(c0, rl.step0);
      c1 = cmul(c1, rl.step1);
    }
  }
}

// Rotates the 16 rows this thread owns in BOTH Q tiles of a unit: the two
// heads share every row's angle, so each angle is formed once.  Angles as in
// rotate_tile; with a per-token table (row_cs != nullptr, row r's 32
// (c cos, c sin) pairs at row_cs[16 r .. 16 r + 15] as float4) explicit
// positions read their row's angles instead of forming them.
__device__ __forceinline__ void rotate_q_pair(const FwdParams& p, const RopeLane& rl, uint8_t* ta, uint8_t* tb,
                                              float2 c0, float2 c1, int n_valid, const int32_t* pos_row0,
                                              const float4* row_cs, int pb) {
  const bool explicit_pos = pos_row0 != nullptr;
#pragma unroll 4
  for (int kk = 0; kk < 16; ++kk) {
    const int r = rl.ro + 8 * kk;
    if (r < n_valid) {
      if (explicit_pos) {
        if (row_cs != nullptr) {
          const float4 v = __ldg(row_cs + 16 * r + pb);
          c0 = make_float2(v.x, v.y);
          c1 = make_float2(v.z, v.w);
        } else {
          const int pos = __ldg(pos_row0 + r);
          c0 = rope_cs(pos, rl.f0, p.tab.conc);
          c1 = rope_cs(pos, rl.f1, p.tab.conc);
        }
      }
      uint32_t* pa_lo = reinterpret_cast<uint32_t*>(ta + rl.w_lo + kk * 1024);
      uint32_t* pa_hi = reinterpret_cast<uint32_t*>(ta + rl.w_hi + kk * 1024);
      uint32_t* pb_lo = reinterpret_cast<uint32_t*>(tb + rl.w_lo + kk * 1024);
      uint32_t* pb_hi = reinterpret_cast<uint32_t*>(tb + rl.w_hi + kk * 1024);
      uint32_t alo = *pa_lo, ahi = *pa_hi, blo = *pb_lo, bhi = *pb_hi;
      rotate_words(alo, ahi, c0, c1);
      rotate_words(blo, bhi, c0, c1);
      *pa_lo = alo;
      *pa_hi = ahi;
      *pb_lo = blo;
      *pb_hi = bhi;
    }
    if (!explicit_pos) {
      c0 = cmul(c0, rl.step0);
      c1 = cmul(c1, rl.step1);
    }
  }
}

__device__ __forceinline__ void fwd_rope_role(const FwdParams& p, FwdSmem& sm) {
  const int rt = threadIdx.x;  // warps 0-3
  const int w = rt >> 5, l = rt & 31;
  const int pb = l & 15;
  RopeLane rl;
  rl.ro = w + 4 * (l >> 4);
  const int e0 = 2 * pb;
  rl.w_lo = sw128_word(rl.ro, e0);
  rl.w_hi = sw128_word(rl.ro, e0 + 32);
  rl.f0 = p.tab.inv_freq[e0];
  rl.f1 = p.tab.inv_freq[e0 + 1];
  const bool rot = p.tab.enabled != 0;
  const bool explicit_pos = p.positions != nullptr;
  const bool thd = p.cu_seqlens != nullptr;
  rl.step0 = rl.step1 = make_float2(1.f, 0.f);
  float2 tstep0 = rl.step0, tstep1 = rl.step1;  // (cos 128f, sin 128f): one tile further
  if (rot && !explicit_pos) {
    rl.step0 = rope_cs(8, rl.f0, 1.f);
    rl.step1 = rope_cs(8, rl.f1, 1.f);
    tstep0 = rope_cs(kFwdTile, rl.f0, 1.f);
    tstep1 = rope_cs(kFwdTile, rl.f1, 1.f);
  }
  const float2 one = make_float2(1.f, 0.f);
  uint32_t i = 0, kv_it = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qb = i & 1;
    const int32_t* pos_seq =
        explicit_pos ? p.positions + (thd ? wu.seq_start : static_cast<int64_t>(wu.b) * p.S) : nullptr;
    // ---- the unit's two Q tiles ----
    if (!mbar_wait_warp_relaxed(&sm.q_loaded[qb], (i >> 1) & 1, p.wait_ns)) return;
    if (rot) {
      const int n_valid = min(kFwdTile, wu.L - wu.q0);
      // the unit's first query token; its rows' angles in the per-token table
      const int64_t tok_q0 = (thd ? wu.seq_start : static_cast<int64_t>(wu.b) * p.S) + wu.q0;
      const float4* row_cs = p.cs_tab != nullptr ? reinterpret_cast<const float4*>(p.cs_tab + tok_q0 * kPairs) : nullptr;
      float2 c0 = one, c1 = one;
      if (!explicit_pos && rl.ro < n_valid) {  // one seed for row ro serves both heads' tiles
        if (row_cs != nullptr) {  // (a thread without a valid row rotates nothing and reads no table row)
          const float4 v = __ldg(row_cs + 16 * rl.ro + pb);
          c0 = make_float2(v.x, v.y);
          c1 = make_float2(v.z, v.w);
        } else {
          c0 = rope_cs(wu.q0 + rl.ro, rl.f0, p.tab.conc);
          c1 = rope_cs(wu.q0 + rl.ro, rl.f1, p.tab.conc);
        }
      }
      rotate_q_pair(p, rl, sm.q[qb][0], sm.q[qb][1], c0, c1, n_valid, explicit_pos ? pos_seq + wu.q0 : nullptr,
                    row_cs, pb);
      fence_proxy_async_smem();
    }
    mbar_arrive(&sm.q_full[qb]);
    ++i;
    if (!p.k_in_kernel) continue;  // k arrives rotated (or RoPE is off): QK^T waits on the copy itself
    // ---- the unit's K tiles: consecutive, so one seed plus a fixed step each ----
    float2 k0s = one, k1s = one;
    if (!explicit_pos) {
      k0s = rope_cs(wu.j_lo * kFwdTile + rl.ro, rl.f0, p.tab.conc);
      k1s = rope_cs(wu.j_lo * kFwdTile + rl.ro, rl.f1, p.tab.conc);
    }
    for (int j = 0; j < wu.n_kt; ++j, ++kv_it) {
      const int s = kv_it % kFwdStages;
      if (!mbar_wait_warp_relaxed(&sm.k_full[s], (kv_it / kFwdStages) & 1, p.wait_ns)) return;
      {
        const int k0 = (wu.j_lo + j) * kFwdTile;
        rotate_tile(p, rl, sm.k[s], k0s, k1s, min(kFwdTile, wu.L - k0), explicit_pos ? pos_seq + k0 : nullptr);
        fence_proxy_async_smem();
        k0s = cmul(k0s, tstep0);
        k1s = cmul(k1s, tstep1);
      }
      mbar_arrive(&sm.k_ready[s]);
    }
  }
}

}  // namespace gptoss
