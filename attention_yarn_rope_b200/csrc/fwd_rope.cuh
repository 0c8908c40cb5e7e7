// fwd_rope.cuh -- rope warpgroup of the prefill kernel: RoPE fused into the
// Q tile load (NeMo AutoModel gpt_oss.rope_utils page, apply_rotary_emb_qk:
// half-split pairs, concentration applied).
//
// TMA lands the raw bf16 Q tiles of a unit (two heads, 128 rows x 64
// features each, 128B-swizzled) in shared memory; this warpgroup rotates
// them in place and leaves fp16 values for the QK^T product (k arrives
// rotated, in fp16, from the call's first kernel).  Without RoPE the same
// pass only converts bf16 to fp16: the host then supplies the identity table
// (every angle 0, concentration 1), so each value is multiplied by exactly 1.
//
// With R = rotary_dim / 2 rotary pairs (j, j + R), thread (w, l), pb = l % 16,
// owns two 32-bit words (feature pairs) of rows ro, ro+8, ..., ro+120 with
// ro = w + 4 (l / 16) -- the two half-warps touch rows 4 apart, whose
// swizzled chunks fall in disjoint banks.  For pb < R/2 they are words pb
// and pb + R/2, i.e. pairs (2pb, 2pb+R) and (2pb+1, 2pb+1+R), rotated; the
// other threads own words 2pb and 2pb+1 past the rotary features (partial
// rotary), which are only converted (angle 0, no concentration).  R = 32
// (GPT-OSS) leaves no pass-through words.  The angle of row ro + 8k is the
// row-ro seed times (cos 8f, sin 8f)^k: one seed per tile and pair (from the
// per-token table the first kernel wrote), the rest complex
// multiplications, so no transcendental per element.  With explicit
// positions every row reads its own angles from that table.
#pragma once

#include "fwd_common.cuh"

namespace gptoss {

struct RopeLane {
  int ro;                 // first row of this thread
  uint32_t w_lo, w_hi;    // byte offsets of its two words in row ro
  float2 step0, step1;    // (cos 8f, sin 8f) of its two pairs
  bool rotates;           // false: the words lie past the rotary features
};

// Rotates the 16 rows this thread owns in BOTH Q tiles of a unit: the two
// heads share every row's angle, so each angle is formed once.  (c0, c1) is
// the angle of row ro for the thread's two pairs, concentration included;
// row ro + 8k gets (c, s) * (cos 8f, sin 8f)^k.  With explicit positions
// (row_cs != nullptr and per_row) row r's 32 (c cos, c sin) pairs are read at
// row_cs[16 r .. 16 r + 15] as float4.  Rows at or past n_valid (beyond the
// sequence) are only converted to fp16: their scores are masked, but their
// bits must be fp16 numbers, not bf16 ones read as fp16.  (Measured: a rolled
// loop, row by row, beats 4-way unrolling by 5 % on the sliding window -- the
// softmax warps' code shares the instruction cache -- and beats loading all
// 32 words up front.)
__device__ __forceinline__ void rotate_q_pair(const RopeLane& rl, uint8_t* ta, uint8_t* tb, float2 c0, float2 c1,
                                              int n_valid, bool per_row, const float4* row_cs, int pb) {
  const float2 one = make_float2(1.f, 0.f);
#pragma unroll 1
  for (int kk = 0; kk < 16; ++kk) {
    const int r = rl.ro + 8 * kk;
    float2 a0 = one, a1 = one;
    if (r < n_valid && rl.rotates) {
      if (per_row) {
        const float4 v = __ldg(row_cs + 16 * r + pb);
        a0 = make_float2(v.x, v.y);
        a1 = make_float2(v.z, v.w);
      } else {
        a0 = c0;
        a1 = c1;
      }
    }
    uint32_t* pa_lo = reinterpret_cast<uint32_t*>(ta + rl.w_lo + kk * 1024);
    uint32_t* pa_hi = reinterpret_cast<uint32_t*>(ta + rl.w_hi + kk * 1024);
    uint32_t* pb_lo = reinterpret_cast<uint32_t*>(tb + rl.w_lo + kk * 1024);
    uint32_t* pb_hi = reinterpret_cast<uint32_t*>(tb + rl.w_hi + kk * 1024);
    uint32_t alo = *pa_lo, ahi = *pa_hi, blo = *pb_lo, bhi = *pb_hi;
    rotate_words(alo, ahi, a0, a1);
    rotate_words(blo, bhi, a0, a1);
    *pa_lo = alo;
    *pa_hi = ahi;
    *pb_lo = blo;
    *pb_hi = bhi;
    if (!per_row) {
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
  const int R = p.tab.R;
  rl.rotates = 2 * pb < R;
  const int e0 = 2 * pb;
  rl.w_lo = sw128_word(rl.ro, rl.rotates ? e0 : 4 * pb);
  rl.w_hi = sw128_word(rl.ro, rl.rotates ? e0 + R : 4 * pb + 2);
  const bool explicit_pos = p.positions != nullptr;
  const bool thd = p.cu_seqlens != nullptr;
  rl.step0 = rope_cs(8, rl.rotates ? p.tab.inv_freq[e0] : 0.0, 1.f);
  rl.step1 = rope_cs(8, rl.rotates ? p.tab.inv_freq[e0 + 1] : 0.0, 1.f);
  const float2 one = make_float2(1.f, 0.f);
  uint32_t i = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qb = i % kFwdQStages;
    if (!mbar_wait_warp_relaxed(&sm.q_loaded[qb], (i / kFwdQStages) & 1, p.wait_ns)) return;
    const int n_valid = min(kFwdTile, wu.L - wu.q0);
    // the unit's first query token; its rows' angles in the per-token table
    const int64_t tok_q0 = (thd ? wu.seq_start : static_cast<int64_t>(wu.b) * p.S) + wu.q0;
    const float4* row_cs = reinterpret_cast<const float4*>(p.cs_tab + tok_q0 * kPairs);
    float2 c0 = one, c1 = one;
    if (!explicit_pos && rl.ro < n_valid && rl.rotates) {  // one seed for row ro serves both heads' tiles
      const float4 v = __ldg(row_cs + 16 * rl.ro + pb);
      c0 = make_float2(v.x, v.y);
      c1 = make_float2(v.z, v.w);
    }
    rotate_q_pair(rl, sm.q[qb][0], sm.q[qb][1], c0, c1, n_valid, explicit_pos, row_cs, pb);
    fence_proxy_async_smem();
    mbar_arrive(&sm.q_full[qb]);
    ++i;
  }
}

}  // namespace gptoss
