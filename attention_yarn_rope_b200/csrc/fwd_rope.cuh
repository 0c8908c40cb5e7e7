// fwd_rope.cuh -- rope warpgroup of the prefill kernel: RoPE fused into the
// Q and K tile loads (NeMo AutoModel gpt_oss.rope_utils page,
// apply_rotary_emb_qk: half-split pairs, concentration applied).
//
// Thread (w, l) owns pairs (2pb, 2pb+32) and (2pb+1, 2pb+33), pb = l % 16, of
// rows ro, ro+8, ..., ro+120 with ro = w + 4 (l / 16): the two half-warps
// touch rows 4 apart, whose 128B-swizzled chunks fall in disjoint banks.  The
// angle of row ro + 8k is the row-ro seed times (cos 8f, sin 8f)^k: one
// double-precision seed per tile and pair (rope_cs), the rest complex
// multiplications, so no transcendental per element.  With explicit
// positions every row gets its own seed.
#pragma once

#include "fwd_common.cuh"

namespace gptoss {

__device__ __forceinline__ void fwd_rope_role(const FwdParams& p, FwdSmem& sm) {
  const int rt = threadIdx.x - 256;
  const int w = rt >> 5, l = rt & 31;
  const int pb = l & 15;
  const int ro = w + 4 * (l >> 4);
  const int e0 = 2 * pb;
  const uint32_t w_lo = sw128_word(ro, e0), w_hi = sw128_word(ro, e0 + 32);  // + 1024 per 8 rows
  const bool rot = p.tab.enabled != 0;
  const bool explicit_pos = p.positions != nullptr;
  const bool thd = p.cu_seqlens != nullptr;
  const double f0 = p.tab.inv_freq[e0], f1 = p.tab.inv_freq[e0 + 1];
  float2 step0 = make_float2(1.f, 0.f), step1 = make_float2(1.f, 0.f);
  if (rot && !explicit_pos) {
    step0 = rope_cs(8, f0, 1.f);
    step1 = rope_cs(8, f1, 1.f);
  }
  uint32_t i = 0, kv_it = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qb = i & 1;
    if (!mbar_wait_warp(&sm.q_empty[qb], ((i >> 1) & 1) ^ 1, p.wait_ns)) return;
    const int64_t pos_base = thd ? wu.seq_start : static_cast<int64_t>(wu.b) * p.S;
    // ---- the unit's two Q tiles: raw rows -> rotated, swizzled shared memory ----
#pragma unroll 1
    for (int X = 0; X < 2; ++X) {
      const int h = X == 0 ? wu.h0 : wu.h1;
      uint8_t* qs = sm.q[qb][X];
      float2 c0 = make_float2(1.f, 0.f), c1 = c0;
      if (rot && !explicit_pos) {
        c0 = rope_cs(wu.q0 + ro, f0, p.tab.conc);
        c1 = rope_cs(wu.q0 + ro, f1, p.tab.conc);
      }
#pragma unroll 4
      for (int kk = 0; kk < 16; ++kk) {
        const int qi = wu.q0 + ro + 8 * kk;
        uint32_t lo = 0, hi = 0;
        if (qi < wu.L) {
          const int64_t row = thd ? static_cast<int64_t>(wu.seq_start + qi) * p.sq.tok
                                  : static_cast<int64_t>(wu.b) * p.sq.batch + static_cast<int64_t>(qi) * p.sq.tok;
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
    }
    fence_proxy_async_smem();
    mbar_arrive(&sm.q_full[qb]);
    // ---- the unit's K tiles: rotate in place once TMA has landed them ----
    for (int j = 0; j < wu.n_kt; ++j, ++kv_it) {
      const int s = kv_it % kFwdStages;
      if (!mbar_wait_warp(&sm.k_full[s], (kv_it / kFwdStages) & 1, p.wait_ns)) return;
      if (rot) {
        uint8_t* ks = sm.k[s];
        const int k0 = (wu.j_lo + j) * kFwdTile;
        float2 c0 = make_float2(1.f, 0.f), c1 = c0;
        if (!explicit_pos) {
          c0 = rope_cs(k0 + ro, f0, p.tab.conc);
          c1 = rope_cs(k0 + ro, f1, p.tab.conc);
        }
#pragma unroll 4
        for (int kk = 0; kk < 16; ++kk) {
          const int key = k0 + ro + 8 * kk;
          if (key < wu.L) {
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
    ++i;
  }
}

}  // namespace gptoss
