// attn_fwd.cuh -- prefill sink attention with fused YaRN RoPE (gptoss_attn_fwd).
//
// Rule: GptOssAttention on the NeMo AutoModel gpt_oss.layers page (sinks,
// sliding_window, softmax_scale = head_dim^-0.5, grouped query heads), RoPE of
// the gpt_oss.rope_utils page, sink in the denominator only (Transformers
// v4.55.0 release notes, "Architecture").
//
// Design (one CTA per 128-query tile of one (sequence, q-head), 10 warps):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r; reads S from
//              TMEM, masks boundary tiles, online softmax in log2 units with
//              the sink folded into the initial running max / sum, writes P
//              (bf16) back into TMEM over S, rescales O in TMEM when the
//              running max moved by more than 2^8, final O / l epilogue.
//   warps 4-7  rope: loads the raw Q tile, rotates it and writes it to shared
//              memory in the 128B-swizzled layout the tensor core reads; then
//              rotates every K tile in place after TMA lands it (angles by
//              complex recurrence along the rows: one seed per tile and pair,
//              so no transcendental per element).
//   warp 8     TMA producer: K and V tiles (128 keys x 64) into a 4-stage ring.
//   warp 9     allocates TMEM (512 columns) and issues tcgen05.mma:
//              S[buf] = Q K^T (SS, M128 N128 K16 x4) into one of two S buffers,
//              then O += P V (TS: P from TMEM, V from shared memory, M128 N64
//              K16 x8), with tcgen05.commit signalling every consumer.
// Key tiles entirely outside the causal band or the sliding window are never
// loaded; only tiles crossing the diagonal, the window edge or the end of
// the sequence are masked.
#pragma once

#include "host_util.cuh"
#include "rope_qk.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

constexpr int kFwdTile = 128;         // query rows and keys per tile
constexpr int kFwdStages = 4;
constexpr int kFwdThreads = 320;
constexpr int kFwdTileBytes = kFwdTile * kHeadDim * 2;  // 16 KB
constexpr uint32_t kFwdTmemCols = 512;
constexpr uint32_t kTmemO = 256;      // O accumulator columns [256, 320)
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct FwdParams {
  CUtensorMap tmap_k;  // dims (64, Hkv, S or T, B or 1), box (64, 1, 128, 1)
  CUtensorMap tmap_v;
  const __nv_bfloat16* q;
  gptoss_strides sq;
  __nv_bfloat16* out;
  gptoss_strides so;
  float* lse;
  const float* sinks;
  const int32_t* positions;
  const int32_t* cu_seqlens;
  int B, S, T, Hq, Hkv, G, window, n_qtiles;
  float scale_log2;
  uint64_t wait_ns;
  RopeTable tab;
};

struct __align__(1024) FwdSmem {
  uint8_t q[kFwdTileBytes];
  uint8_t k[kFwdStages][kFwdTileBytes];
  uint8_t v[kFwdStages][kFwdTileBytes];
  uint64_t q_full;
  uint64_t k_full[kFwdStages], k_ready[kFwdStages], k_empty[kFwdStages];
  uint64_t v_full[kFwdStages], v_empty[kFwdStages];
  uint64_t s_full[2], p_full[2], s_free[2];
  uint64_t o_done;
  uint64_t mma_final;
  uint32_t tmem_base;
};

// Byte offset of the 32-bit word holding features (e, e+1) of row r in a
// 128B-swizzled 128 x 64 bf16 tile (e even).
__device__ __forceinline__ uint32_t sw128_word(int r, int e) {
  return r * 128 + ((((e >> 3) ^ (r & 7))) << 4) + (e & 7) * 2;
}

// Rotates the two pairs held in words (lo, hi) = features (e, e+1), (e+32, e+33).
__device__ __forceinline__ void rotate_words(uint32_t& lo, uint32_t& hi, float2 a, float2 b) {
  const float x0 = bf16lo(lo), x1 = bf16hi(lo);
  const float y0 = bf16lo(hi), y1 = bf16hi(hi);
  lo = pack_bf16(x0 * a.x - y0 * a.y, x1 * b.x - y1 * b.y);
  hi = pack_bf16(y0 * a.x + x0 * a.y, y1 * b.x + x1 * b.y);
}

// (c, s) <- (c, s) * (cos d, sin d): advances an angle seed by a fixed step.
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}

__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  // ---- work unit: heaviest query tiles first ----
  const int per_tile = p.Hq * p.B;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / per_tile;
  const int rest = static_cast<int>(blockIdx.x) % per_tile;
  const int h = rest % p.Hq;
  const int b = rest / p.Hq;
  const int g = h / p.G;
  const bool thd = p.cu_seqlens != nullptr;
  const int seq_start = thd ? __ldg(p.cu_seqlens + b) : 0;
  const int L = thd ? __ldg(p.cu_seqlens + b + 1) - seq_start : p.S;
  const int q0 = qt * kFwdTile;
  if (q0 >= L) return;  // past the end of this packed sequence
  const int q_last = min(q0 + kFwdTile, L) - 1;
  const int j_hi = q_last / kFwdTile;
  const int j_lo = p.window > 0 ? max(0, q0 - p.window + 1) / kFwdTile : 0;
  const int n_kt = j_hi - j_lo + 1;

  extern __shared__ uint8_t smem_raw[];
  FwdSmem& sm = *reinterpret_cast<FwdSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 128);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_ready[s], 128);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.s_free[i], 1);
    }
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.mma_final, 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // token coordinate (4-D tensor-map row) of key tile j
  const int tok_row0 = thd ? seq_start : 0;
  const int bcoord = thd ? 0 : b;

  if (warp < 4) {
    // ====================== softmax warpgroup ======================
    const int r = threadIdx.x;  // query row within the tile, TMEM lane
    const int qi = q0 + r;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sink = __ldg(p.sinks + h) * kLog2e;
    float m_run = sink;                       // running max, log2 units
    float l_run = sink == -INFINITY ? 0.f : 1.f;  // exp2(sink - m_run)
    bool ok = true;
    for (int it = 0; it < n_kt && ok; ++it) {
      const int buf = it & 1;
      const int j = j_lo + it;
      const int k0 = j * kFwdTile;
      if (!mbar_wait_warp(&sm.s_full[buf], (it >> 1) & 1, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + buf * 128 + c * 32, sr[c]);
      tmem_wait_ld();
      // visible columns of this row: [c_lo, c_hi]
      const bool edge = (k0 + kFwdTile - 1 > q0) || (p.window > 0 && q0 + kFwdTile - 1 - k0 >= p.window) ||
                        (k0 + kFwdTile - 1 >= L);
      float mt = -INFINITY;
      if (edge) {
        const int c_hi = min(qi, L - 1) - k0;
        const int c_lo = p.window > 0 ? qi - p.window + 1 - k0 : -1;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int col = c * 32 + e;
            float x = __uint_as_float(sr[c][e]);
            x = (col <= c_hi && col >= c_lo) ? x : -INFINITY;
            sr[c][e] = __float_as_uint(x);
            mt = fmaxf(mt, x);
          }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) mt = fmaxf(mt, __uint_as_float(sr[c][e]));
      }
      const float m_cand = mt * p.scale_log2;
      float alpha = 1.f;
      bool rescale = false;
      if (m_cand > m_run + kRescaleThreshold) {
        alpha = ex2_approx(m_run - m_cand);  // 0 when m_run == -inf
        m_run = m_cand;
        rescale = true;
      }
      const float base = m_run == -INFINITY ? 0.f : m_run;
      float rs = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int w = 0; w < 32; ++w) {
          const int col = half * 64 + 2 * w;
          const float x0 = ex2_approx(fmaf(__uint_as_float(sr[col >> 5][col & 31]), p.scale_log2, -base));
          const float x1 = ex2_approx(fmaf(__uint_as_float(sr[(col + 1) >> 5][(col + 1) & 31]), p.scale_log2, -base));
          rs += x0 + x1;
          pk[w] = pack_bf16(x0, x1);
        }
        tmem_st32(lane_base + buf * 128 + half * 32, pk);
      }
      l_run = l_run * alpha + rs;
      tmem_wait_st();
      if (it > 0) {
        // O is stable only once the previous P V product has completed
        if (!mbar_wait_warp(&sm.o_done, (it - 1) & 1, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (rescale) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t ov[32];
            tmem_ld32(lane_base + kTmemO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(lane_base + kTmemO + c * 32, ov);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.p_full[buf]);
    }
    // ---- epilogue: O / l, LSE ----
    if (ok && mbar_wait_warp(&sm.o_done, (n_kt - 1) & 1, p.wait_ns)) {
      tc_fence_after();
      uint32_t ov[2][32];
      tmem_ld32(lane_base + kTmemO, ov[0]);
      tmem_ld32(lane_base + kTmemO + 32, ov[1]);
      tmem_wait_ld();
      if (qi < L) {
        const float inv = 1.f / l_run;
        const int64_t row = thd ? static_cast<int64_t>(seq_start + qi) * p.so.tok
                                : static_cast<int64_t>(b) * p.so.batch + static_cast<int64_t>(qi) * p.so.tok;
        __nv_bfloat16* dst = p.out + row + static_cast<int64_t>(h) * p.so.head;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint4 v;
          const int c = c8 >> 2, e = (c8 & 3) * 8;
          v.x = pack_bf16(__uint_as_float(ov[c][e + 0]) * inv, __uint_as_float(ov[c][e + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(ov[c][e + 2]) * inv, __uint_as_float(ov[c][e + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(ov[c][e + 4]) * inv, __uint_as_float(ov[c][e + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(ov[c][e + 6]) * inv, __uint_as_float(ov[c][e + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + c8 * 8) = v;
        }
        if (p.lse != nullptr) {
          const float lse = (m_run + log2f(l_run)) * kLn2;
          if (thd)
            p.lse[static_cast<int64_t>(h) * p.T + seq_start + qi] = lse;
          else
            p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.S + qi] = lse;
        }
      }
    }
  } else if (warp < 8) {
    // ====================== rope warpgroup ======================
    const int rt = threadIdx.x - 128;
    const int w = rt >> 5, l = rt & 31;
    const int pb = l & 15;            // owns pairs (2pb, 2pb+32) and (2pb+1, 2pb+33)
    const int ro = w + 4 * (l >> 4);  // rows ro, ro+8, ..., ro+120
    const int e0 = 2 * pb;
    const uint32_t w_lo = sw128_word(ro, e0), w_hi = sw128_word(ro, e0 + 32);  // + 1024 per 8 rows
    const bool rot = p.tab.enabled != 0;
    const bool explicit_pos = p.positions != nullptr;
    const double f0 = p.tab.inv_freq[e0], f1 = p.tab.inv_freq[e0 + 1];
    float2 step0 = make_float2(1.f, 0.f), step1 = make_float2(1.f, 0.f);
    if (rot && !explicit_pos) {
      step0 = rope_cs(8, f0, 1.f);
      step1 = rope_cs(8, f1, 1.f);
    }
    const int64_t pos_base = thd ? seq_start : static_cast<int64_t>(b) * p.S;  // index into positions
    // ---- Q tile: raw rows from global -> rotated, swizzled shared memory ----
    {
      uint8_t* qs = sm.q;
      float2 c0 = make_float2(1.f, 0.f), c1 = c0;
      if (rot && !explicit_pos) {
        c0 = rope_cs(q0 + ro, f0, p.tab.conc);
        c1 = rope_cs(q0 + ro, f1, p.tab.conc);
      }
#pragma unroll 4
      for (int kk = 0; kk < 16; ++kk) {
        const int r = ro + 8 * kk;
        const int qi = q0 + r;
        uint32_t lo = 0, hi = 0;
        if (qi < L) {
          const int64_t row = thd ? static_cast<int64_t>(seq_start + qi) * p.sq.tok
                                  : static_cast<int64_t>(b) * p.sq.batch + static_cast<int64_t>(qi) * p.sq.tok;
          const __nv_bfloat16* src = p.q + row + static_cast<int64_t>(h) * p.sq.head;
          lo = *reinterpret_cast<const uint32_t*>(src + e0);
          hi = *reinterpret_cast<const uint32_t*>(src + e0 + 32);
          if (rot) {
            if (explicit_pos) {
              const int pos = __ldg(p.positions + pos_base + qi);
              c0 = rope_cs(pos, f0, p.tab.conc);
              c1 = rope_cs(pos, f1, p.tab.conc);
            }
            rotate_words(lo, hi, c0, c1);
          }
        }
        if (rot && !explicit_pos) {
          c0 = cmul(c0, step0);
          c1 = cmul(c1, step1);
        }
        *reinterpret_cast<uint32_t*>(qs + w_lo + kk * 1024) = lo;
        *reinterpret_cast<uint32_t*>(qs + w_hi + kk * 1024) = hi;
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.q_full);
    }
    // ---- K tiles: rotate in place once TMA has landed them ----
    for (int it = 0; it < n_kt; ++it) {
      const int s = it % kFwdStages;
      if (!mbar_wait_warp(&sm.k_full[s], (it / kFwdStages) & 1, p.wait_ns)) break;
      if (rot) {
        uint8_t* ks = sm.k[s];
        const int k0 = (j_lo + it) * kFwdTile;
        float2 c0 = make_float2(1.f, 0.f), c1 = c0;
        if (!explicit_pos) {
          c0 = rope_cs(k0 + ro, f0, p.tab.conc);
          c1 = rope_cs(k0 + ro, f1, p.tab.conc);
        }
#pragma unroll 4
        for (int kk = 0; kk < 16; ++kk) {
          const int key = k0 + ro + 8 * kk;
          if (key < L) {
            if (explicit_pos) {
              const int pos = __ldg(p.positions + pos_base + key);
              c0 = rope_cs(pos, f0, p.tab.conc);
              c1 = rope_cs(pos, f1, p.tab.conc);
            }
            uint32_t* plo = reinterpret_cast<uint32_t*>(ks + w_lo + kk * 1024);
            uint32_t* phi = reinterpret_cast<uint32_t*>(ks + w_hi + kk * 1024);
            uint32_t lo = *plo, hi = *phi;
            rotate_words(lo, hi, c0, c1);
            *plo = lo;
            *phi = hi;
          }
          if (!explicit_pos) {
            c0 = cmul(c0, step0);
            c1 = cmul(c1, step1);
          }
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&sm.k_ready[s]);
    }
  } else if (warp == 8) {
    // ====================== TMA producer ======================
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_k);
      tma_prefetch_desc(&p.tmap_v);
      int k_issued = 0, v_issued = 0;
      for (int it = 0; it < n_kt; ++it) {
        const int s = it % kFwdStages;
        const uint32_t ph = ((it / kFwdStages) & 1) ^ 1;
        const int key_row = tok_row0 + (j_lo + it) * kFwdTile;
        if (!mbar_wait(&sm.k_empty[s], ph, p.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.k_full[s], kFwdTileBytes);
        tma_load_4d(sm.k[s], &p.tmap_k, &sm.k_full[s], 0, g, key_row, bcoord);
        k_issued = it + 1;
        if (!mbar_wait(&sm.v_empty[s], ph, p.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.v_full[s], kFwdTileBytes);
        tma_load_4d(sm.v[s], &p.tmap_v, &sm.v_full[s], 0, g, key_row, bcoord);
        v_issued = it + 1;
      }
      // drain: the copies of the last stages must land before the CTA exits
      for (int it = max(0, k_issued - kFwdStages); it < k_issued; ++it)
        mbar_wait(&sm.k_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
      for (int it = max(0, v_issued - kFwdStages); it < v_issued; ++it)
        mbar_wait(&sm.v_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
    }
  } else {
    // ====================== MMA issuer ======================
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, 64, true);
      const uint64_t qdesc = sw128_desc(smem_u32(sm.q));
      bool ok = mbar_wait(&sm.q_full, 0, p.wait_ns);
      int pv_issued = 0;
      auto issue_pv = [&](int i) -> bool {
        const int buf = i & 1, s = i % kFwdStages;
        if (!mbar_wait(&sm.p_full[buf], (i >> 1) & 1, p.wait_ns)) return false;
        if (!mbar_wait(&sm.v_full[s], (i / kFwdStages) & 1, p.wait_ns)) return false;
        tc_fence_after();
        const uint64_t vdesc = sw128_desc(smem_u32(sm.v[s]));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + kTmemO, tmem + buf * 128 + kk * 8, vdesc + static_cast<uint64_t>(kk * 128), idesc_o,
                 (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.v_empty[s]);
        mma_commit(&sm.s_free[buf]);
        mma_commit(&sm.o_done);
        pv_issued = i + 1;
        return true;
      };
      for (int it = 0; it < n_kt && ok; ++it) {
        const int buf = it & 1, s = it % kFwdStages;
        if (!mbar_wait(&sm.k_ready[s], (it / kFwdStages) & 1, p.wait_ns)) { ok = false; break; }
        if (it >= 2 && !mbar_wait(&sm.s_free[buf], ((it >> 1) + 1) & 1, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s]));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + buf * 128, qdesc + static_cast<uint64_t>(kk * 2), kdesc + static_cast<uint64_t>(kk * 2),
                 idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(&sm.k_empty[s]);
        mma_commit(&sm.s_full[buf]);
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(n_kt - 1);
      // every issued MMA must finish before TMEM is released
      mma_commit(&sm.mma_final);
      mbar_wait(&sm.mma_final, 0, p.wait_ns);
      (void)pv_issued;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace gptoss
