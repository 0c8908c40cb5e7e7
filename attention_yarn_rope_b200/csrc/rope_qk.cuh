// rope_qk.cuh -- standalone YaRN RoPE of q and k (gptoss_rope_qk).
//
// Rule: NeMo AutoModel gpt_oss.rope_utils page, apply_rotary_emb_qk /
// _apply_rotary_emb_qk: q and k rotated with the same tables, half-split
// pairs (j, j + R) with R = rotary_dim / 2, concentration applied, features
// from rotary_dim on passed through unchanged (apply_rotary_emb, partial
// rotary), BSHD or packed THD with cu_seqlens.
//
// Design (HBM-bound elementwise op): a CTA owns TB consecutive tokens.  Its
// threads first build the (c cos, c sin) table of those tokens' R angles in
// shared memory -- the angle p * inv_freq is formed and reduced modulo 2 pi
// in double precision, then sincosf runs on the reduced angle -- and then
// sweep every (token, head, 16-byte chunk) of q and k with 128-bit loads and
// stores.  A rotation item takes chunk c (features [8c, 8c+8)) and its
// partner chunk c + R/8 (features [R+8c, R+8c+8)): 8 complete pairs; a
// pass-through item copies one chunk past 2R.  R = 32 (GPT-OSS) gives 4
// rotation items per head: a warp covers 8 heads x 4 items of one token, so
// its two loads fill whole 128-byte lines.  Head size D is 64 or 128 (D / 8
// chunks per head row, R <= D / 2).
#pragma once

#include "host_util.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

struct TokenMap {
  const int32_t* positions;   // nullable
  const int32_t* cu_seqlens;  // nullable -> BSHD
  int nseq;                   // THD: number of sequences; BSHD: B
  int S;                      // BSHD sequence length
  int ntok;                   // B*S or T
  int pos_offset;             // default positions: index in the sequence + pos_offset
};

// Token t -> (batch row or sequence, index inside it).
__device__ __forceinline__ void token_coords(const TokenMap& m, int t, int& seq, int& idx) {
  if (m.cu_seqlens == nullptr) {
    seq = t / m.S;
    idx = t - seq * m.S;
  } else {
    int lo = 0, hi = m.nseq - 1;  // last sequence whose start <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(m.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
    }
    seq = lo;
    idx = t - __ldg(m.cu_seqlens + lo);
    // cu_seqlens nondecreasing around t: cu[lo] <= t < cu[lo + 1]
    if (!index_ok(idx >= 0 && (lo + 1 > m.nseq || t < __ldg(m.cu_seqlens + lo + 1)))) idx = 0;
  }
}

// The two features of rotation slot j (0 <= j < 32) with R rotary pairs:
// slot j < R is the pair (j, j + R); slots j >= R cover the features past
// the rotary ones, two each (2j, 2j + 1), which pass through unrotated.
__host__ __device__ __forceinline__ int rope_feature_a(int j, int R) { return j < R ? j : 2 * j; }
__host__ __device__ __forceinline__ int rope_feature_b(int j, int R) { return j < R ? j + R : 2 * j + 1; }

// (c cos theta, c sin theta), theta = pos * f, reduced modulo 2 pi in double
// (Cody-Waite with 2 pi split in two doubles), then sincosf on |r| <= pi.
__device__ __forceinline__ float2 rope_cs(int pos, double f, float conc) {
  const double kTwoPiHi = 6.283185307179586;        // nearest double to 2 pi
  const double kTwoPiLo = 2.4492935982947064e-16;   // 2 pi - kTwoPiHi
  const double kInvTwoPi = 0.15915494309189535;     // 1 / (2 pi)
  const double th = static_cast<double>(pos) * f;
  const double k = rint(th * kInvTwoPi);
  double r = fma(-k, kTwoPiHi, th);
  r = fma(-k, kTwoPiLo, r);
  float s, c;
  sincosf(static_cast<float>(r), &s, &c);
  return make_float2(c * conc, s * conc);
}

// Rotates the 8 pairs held by (lo, hi): lo = features [8c, 8c+8), hi = the
// partners [R+8c, R+8c+8); cs[e] = (c cos, c sin) of pair 8c+e.  The result
// is rounded to bf16, or to fp16 when kF16Out (the QK^T operand format of the
// prefill kernel under fused RoPE).
template <bool kF16Out>
__device__ __forceinline__ void rotate8(uint4& lo, uint4& hi, const float2* cs) {
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float x0 = bf16lo(l[w]), x1 = bf16hi(l[w]);
    const float y0 = bf16lo(h[w]), y1 = bf16hi(h[w]);
    const float2 a = cs[2 * w], b = cs[2 * w + 1];
    const float rx0 = x0 * a.x - y0 * a.y, rx1 = x1 * b.x - y1 * b.y;
    const float ry0 = y0 * a.x + x0 * a.y, ry1 = y1 * b.x + x1 * b.y;
    l[w] = kF16Out ? pack_f16(rx0, rx1) : pack_bf16(rx0, rx1);
    h[w] = kF16Out ? pack_f16(ry0, ry1) : pack_bf16(ry0, ry1);
  }
}

struct RopeQkParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_out;
  gptoss_strides sq, sk, sqo, sko;
  const __nv_bfloat16* v;  // nullable: v copied unrotated to v_out (in the output format)
  __nv_bfloat16* v_out;
  gptoss_strides sv, svo;
  TokenMap tm;
  int Hq, Hkv;
  int D;           // head size: 64 or 128
  RopeTable tab;
  float2* cs_out;  // nullable: each token's D / 2 (c cos, c sin) pairs, [token][D / 2]
};

// Converts 8 bf16 values to fp16 (round to nearest even; exact for the
// values fp16 represents).
__device__ __forceinline__ void bf16x8_to_f16(uint4& x) {
  uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = pack_f16(bf16lo(w[i]), bf16hi(w[i]));
}

constexpr int kRopeTokensPerCta = 8;
constexpr int kRopeThreads = 256;

// q (Hq heads, may be 0) and k (Hkv heads) of TB tokens per CTA, and v
// (Hkv heads, unrotated) when p.v is set.  kF16Out: fp16 results (k rotated
// and v converted once for the prefill kernel); otherwise bf16.
template <bool kF16Out>
__global__ void __launch_bounds__(kRopeThreads) rope_qk_kernel(const __grid_constant__ RopeQkParams p) {
  constexpr int TB = kRopeTokensPerCta;
  __shared__ float2 tab[TB][kMaxPairs];
  __shared__ int64_t tok_off[TB][6];  // element offsets of token rows: q, k, q_out, k_out, v, v_out
  const int t0 = blockIdx.x * TB;
  const int tid = threadIdx.x;
  const int np = p.D / 2;  // table entries per token
  for (int ti = tid; ti < TB * np; ti += kRopeThreads) {
    const int tt = ti / np, j = ti % np;
    const int t = t0 + tt;
    if (t < p.tm.ntok) {
      int seq, idx;
      token_coords(p.tm, t, seq, idx);
      const int pos = p.tm.positions ? __ldg(p.tm.positions + t) : idx + p.tm.pos_offset;
      tab[tt][j] = rope_cs(pos, p.tab.inv_freq[j], p.tab.conc);
      if (p.cs_out != nullptr) p.cs_out[static_cast<int64_t>(t) * np + j] = tab[tt][j];
      if (j == 0) {
        const bool thd = p.tm.cu_seqlens != nullptr;
        const int64_t b = thd ? 0 : seq;
        const int64_t s = thd ? t : idx;
        tok_off[tt][0] = b * p.sq.batch + s * p.sq.tok;
        tok_off[tt][1] = b * p.sk.batch + s * p.sk.tok;
        tok_off[tt][2] = b * p.sqo.batch + s * p.sqo.tok;
        tok_off[tt][3] = b * p.sko.batch + s * p.sko.tok;
        tok_off[tt][4] = b * p.sv.batch + s * p.sv.tok;
        tok_off[tt][5] = b * p.svo.batch + s * p.svo.tok;
      }
    }
  }
  __syncthreads();
  const int H = p.Hq + p.Hkv + (p.v != nullptr ? p.Hkv : 0);
  const int n_rot = p.tab.R / 8;     // rotation items per head (chunk + partner)
  const int per_head = p.D / 8 - n_rot;  // plus one pass-through item per chunk past 2R
  const int items = TB * H * per_head;
  for (int it = tid; it < items; it += kRopeThreads) {
    const int ci = it % per_head;
    const int rest = it / per_head;
    const int hh = rest % H;
    const int tt = rest / H;
    if (t0 + tt >= p.tm.ntok) continue;
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    if (hh >= p.Hq + p.Hkv) {  // v: copied in the output format, not rotated
      const int g = hh - p.Hq - p.Hkv;
      src = p.v + tok_off[tt][4] + static_cast<int64_t>(g) * p.sv.head;
      dst = p.v_out + tok_off[tt][5] + static_cast<int64_t>(g) * p.svo.head;
      // the chunks this item would rotate or copy, copied (v is not rotated)
      const int c0 = ci < n_rot ? ci : n_rot + ci;
      const int c1 = ci < n_rot ? ci + n_rot : -1;
      uint4 lo = *reinterpret_cast<const uint4*>(src + 8 * c0);
      if (kF16Out) bf16x8_to_f16(lo);
      *reinterpret_cast<uint4*>(dst + 8 * c0) = lo;
      if (c1 >= 0) {
        uint4 hi = *reinterpret_cast<const uint4*>(src + 8 * c1);
        if (kF16Out) bf16x8_to_f16(hi);
        *reinterpret_cast<uint4*>(dst + 8 * c1) = hi;
      }
      continue;
    }
    if (hh < p.Hq) {
      src = p.q + tok_off[tt][0] + static_cast<int64_t>(hh) * p.sq.head;
      dst = p.q_out + tok_off[tt][2] + static_cast<int64_t>(hh) * p.sqo.head;
    } else {
      const int g = hh - p.Hq;
      src = p.k + tok_off[tt][1] + static_cast<int64_t>(g) * p.sk.head;
      dst = p.k_out + tok_off[tt][3] + static_cast<int64_t>(g) * p.sko.head;
    }
    if (ci < n_rot) {
      uint4 lo = *reinterpret_cast<const uint4*>(src + 8 * ci);
      uint4 hi = *reinterpret_cast<const uint4*>(src + p.tab.R + 8 * ci);
      rotate8<kF16Out>(lo, hi, &tab[tt][8 * ci]);
      *reinterpret_cast<uint4*>(dst + 8 * ci) = lo;
      *reinterpret_cast<uint4*>(dst + p.tab.R + 8 * ci) = hi;
    } else {  // past the rotary features: passed through unchanged
      const int c = n_rot + ci;
      uint4 x = *reinterpret_cast<const uint4*>(src + 8 * c);
      if (kF16Out) bf16x8_to_f16(x);
      *reinterpret_cast<uint4*>(dst + 8 * c) = x;
    }
  }
}

}  // namespace gptoss
