// rope_qk.cuh -- standalone YaRN RoPE of q and k (gptoss_rope_qk).
//
// Rule: NeMo AutoModel gpt_oss.rope_utils page, apply_rotary_emb_qk /
// _apply_rotary_emb_qk: q and k rotated with the same tables, half-split
// pairs (j, j+32), concentration applied, BSHD or packed THD with cu_seqlens.
//
// Design (HBM-bound elementwise op): a CTA owns TB consecutive tokens.  Its
// threads first build the (c cos, c sin) table of those tokens' 32 angles in
// shared memory -- the angle p * inv_freq is formed and reduced modulo 2 pi
// in double precision, then sincosf runs on the reduced angle -- and then
// sweep every (token, head, 16-byte chunk) of q and k with 128-bit loads and
// stores: chunk c of a head holds features [8c, 8c+8) and [32+8c, 40+8c),
// i.e. 8 complete rotation pairs.  A warp covers 8 heads x 4 chunks of one
// token, so its two loads fill whole 128-byte lines.
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
  }
}

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
// partners [32+8c, 40+8c); cs[e] = (c cos, c sin) of pair 8c+e.  The result
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
  TokenMap tm;
  int Hq, Hkv;
  RopeTable tab;
  float2* cs_out;  // nullable: each token's 32 (c cos, c sin) pairs, [token][32]
};

constexpr int kRopeTokensPerCta = 8;
constexpr int kRopeThreads = 256;

// q (Hq heads, may be 0) and k (Hkv heads) of TB tokens per CTA.  kF16Out:
// fp16 results (k rotated once for the prefill kernel); otherwise bf16.
template <bool kF16Out>
__global__ void __launch_bounds__(kRopeThreads) rope_qk_kernel(const __grid_constant__ RopeQkParams p) {
  constexpr int TB = kRopeTokensPerCta;
  __shared__ float2 tab[TB][kPairs];
  __shared__ int64_t tok_off[TB][4];  // element offsets of token rows: q, k, q_out, k_out
  const int t0 = blockIdx.x * TB;
  const int tid = threadIdx.x;
  if (tid < TB * kPairs) {
    const int tt = tid / kPairs, j = tid % kPairs;
    const int t = t0 + tt;
    if (t < p.tm.ntok) {
      int seq, idx;
      token_coords(p.tm, t, seq, idx);
      const int pos = p.tm.positions ? __ldg(p.tm.positions + t) : idx;
      tab[tt][j] = rope_cs(pos, p.tab.inv_freq[j], p.tab.conc);
      if (p.cs_out != nullptr) p.cs_out[static_cast<int64_t>(t) * kPairs + j] = tab[tt][j];
      if (j == 0) {
        const bool thd = p.tm.cu_seqlens != nullptr;
        const int64_t b = thd ? 0 : seq;
        const int64_t s = thd ? t : idx;
        tok_off[tt][0] = b * p.sq.batch + s * p.sq.tok;
        tok_off[tt][1] = b * p.sk.batch + s * p.sk.tok;
        tok_off[tt][2] = b * p.sqo.batch + s * p.sqo.tok;
        tok_off[tt][3] = b * p.sko.batch + s * p.sko.tok;
      }
    }
  }
  __syncthreads();
  const int H = p.Hq + p.Hkv;
  const int items = TB * H * 4;
  for (int it = tid; it < items; it += kRopeThreads) {
    const int chunk = it & 3;
    const int rest = it >> 2;
    const int hh = rest % H;
    const int tt = rest / H;
    if (t0 + tt >= p.tm.ntok) continue;
    const __nv_bfloat16* src;
    __nv_bfloat16* dst;
    if (hh < p.Hq) {
      src = p.q + tok_off[tt][0] + static_cast<int64_t>(hh) * p.sq.head;
      dst = p.q_out + tok_off[tt][2] + static_cast<int64_t>(hh) * p.sqo.head;
    } else {
      const int g = hh - p.Hq;
      src = p.k + tok_off[tt][1] + static_cast<int64_t>(g) * p.sk.head;
      dst = p.k_out + tok_off[tt][3] + static_cast<int64_t>(g) * p.sko.head;
    }
    uint4 lo = *reinterpret_cast<const uint4*>(src + 8 * chunk);
    uint4 hi = *reinterpret_cast<const uint4*>(src + 32 + 8 * chunk);
    rotate8<kF16Out>(lo, hi, &tab[tt][8 * chunk]);
    *reinterpret_cast<uint4*>(dst + 8 * chunk) = lo;
    *reinterpret_cast<uint4*>(dst + 32 + 8 * chunk) = hi;
  }
}

}  // namespace gptoss
