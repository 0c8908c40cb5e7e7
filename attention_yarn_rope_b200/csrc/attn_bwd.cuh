// attn_bwd.cuh -- gradients of the sink attention with RoPE (gptoss_attn_bwd).
//
// Rule: the derivative of GptOssAttention's forward (NeMo AutoModel
// gpt_oss.layers page: sinks, sliding_window, softmax_scale; RoPE of the
// gpt_oss.rope_utils page) for L = sum(dout * out), given the forward's
// log-sum-exp per row (lse includes the sink term).  With P_ij = exp(s_ij -
// lse_i) over the visible pairs and a_i = exp(sink_h - lse_i):
//   D_i = <dout_i, out_i>,  dP_ij = <dout_i, v_j>,  dS_ij = P_ij (dP_ij - D_i)
//   dv_j = sum_i P_ij dout_i,  dq'_i = scale sum_j dS_ij k'_j,
//   dk'_j = scale sum_i dS_ij q'_i,  dsink_h = -sum_i a_i D_i,
// and dq = c R(theta)^T dq', dk = c R(theta)^T dk' (RoPE is linear).
//
// Launches (all on the caller's stream):
//   1. rope_qk_kernel<true>: q and k rotated once into the workspace (fp16,
//      the forward's QK^T operand format) plus each token's 32 (c cos, c sin)
//      pairs; without RoPE the same kernel converts them with the identity.
//   2. attn_bwd_preprocess_kernel: D for every (row, head) into the workspace,
//      and the sink gradient (one atomic add per head and CTA).
//   3. attn_bwd_dkdv_tc_kernel (attn_bwd_tc.cuh): dK and dV on the tcgen05
//      tensor cores, one CTA per (128-key tile, kv head, sequence) sweeping
//      every (query head of the group, 64-query tile) that sees the key tile:
//      S^T = K Q^T, dP^T = V dout^T, P^T and dS^T through tensor memory, dV +=
//      P^T dout, dK += dS^T Q, then scale and c R^T.  A sweep longer than one
//      chunk (full causal: key tile 0 sees every query tile of every head)
//      would leave a few CTAs running long after the rest, so long sweeps are
//      cut into chunks, one CTA each, adding into fp32 dK / dV accumulators;
//      attn_bwd_dkdv_finish_kernel then applies scale and c R^T, writes bf16.
//   4. dQ: attn_bwd_dq_tc_kernel (attn_bwd_tc.cuh, tcgen05) for long sweeps,
//      or attn_bwd_dq_kernel here for short ones (a sliding window): CTA
//      (query tile, head, sequence); 4 warps of 16 queries keep Q and dout as
//      mma.sync A fragments and sweep the key tiles the query tile sees (K and
//      V double-buffered): S, dP, dS recomputed, dQ += dS K, then scale and
//      c R^T.  Recomputing S and dP (3 products per step instead of atomics on
//      a float dQ) keeps every output written once.
// Operands: rotated q / k in fp16, v / dout in bf16, P rounded to bf16 for
// P^T dout and dS to fp16 for the products with q and k; fp32 accumulation.
#pragma once

#include "host_util.cuh"
#include "sm100_ptx.cuh"
#include "warp_mma.cuh"

namespace gptoss {

constexpr int kBwdTile = 64;       // queries / keys per tile
constexpr int kBwdThreads = 128;   // 4 warps x 16 rows
constexpr int kBwdMaxHeads = 1024; // query heads the preprocess kernel reduces in shared memory

struct BwdParams {
  // tensor maps of the tcgen05 dK / dV kernel (dims d, head, token, batch;
  // 128B swizzle): rotated k / q in the workspace (fp16), v and dout (bf16)
  CUtensorMap tmap_k, tmap_v, tmap_q, tmap_do;
  uint64_t wait_ns;         // bound of every device-side wait
  const __nv_bfloat16* qh;  // rotated q, fp16 bits, dense [T, Hq, 64]
  const __nv_bfloat16* kh;  // rotated k, fp16 bits, dense [T, Hkv, 64]
  const __nv_bfloat16* v;
  const __nv_bfloat16* out;
  const __nv_bfloat16* dout;
  gptoss_strides sv, so, sdo;  // elements; BSHD uses batch, THD ignores it
  const float* lse;            // the forward's: BSHD [B, Hq, S], THD [Hq, T]
  float* dsum;                 // D, same layout as lse
  float* lse2;                 // lse log2(e), same layout (the tcgen05 dK / dV kernel's copy)
  const float2* cs;            // [T][32] (c cos, c sin) of every token's pairs
  int R;                       // rotary pairs: features (j, j + R), j < R, rotate; [2R, 64) pass through
  const float* sinks;          // [Hq]
  float* dsinks;               // [Hq], accumulated (zeroed before the launches)
  __nv_bfloat16* dq;           // dense [T, Hq, 64]
  __nv_bfloat16* dk;           // dense [T, Hkv, 64]
  __nv_bfloat16* dv;           // dense [T, Hkv, 64]
  // Split sweeps (max_chunks > 1): a (key tile, kv head) sweep longer than
  // kBwdTcChunkIt steps is cut into chunks, one CTA each, which add their
  // unscaled dK (rotated space) and dV into these fp32 accumulators (zeroed
  // first); attn_bwd_dkdv_finish_kernel then writes dk / dv.
  float* dk_acc;               // [T, Hkv, 64]
  float* dv_acc;               // [T, Hkv, 64]
  int max_chunks;
  const int32_t* cu_seqlens;   // nullable -> BSHD
  int B, S, T, Hq, Hkv, G, window;
  int n_tiles;                 // tiles of the longest sequence
  float scale, scale_log2;
};

struct BwdSeq {
  int64_t tok0;  // dense index of the sequence's first token
  int L;         // its length
};

__device__ __forceinline__ BwdSeq bwd_seq(const BwdParams& p, int b) {
  BwdSeq s;
  if (p.cu_seqlens != nullptr) {
    const int a = __ldg(p.cu_seqlens + b);
    s.tok0 = a;
    s.L = __ldg(p.cu_seqlens + b + 1) - a;
    // cu_seqlens: nondecreasing, within the T tokens, no sequence longer than
    // S; a bad entry makes the sequence empty (skipped)
    if (!index_ok(a >= 0 && s.L >= 0 && a + s.L <= p.T && s.L <= p.S)) {
      s.tok0 = 0;
      s.L = 0;
    }
  } else {
    s.tok0 = static_cast<int64_t>(b) * p.S;
    s.L = p.S;
  }
  return s;
}

// Index of (sequence b, head h, row i) in the lse / D layout.
__device__ __forceinline__ int64_t bwd_row_index(const BwdParams& p, int b, int h, int i, int64_t tok0) {
  return p.cu_seqlens != nullptr ? static_cast<int64_t>(h) * p.T + tok0 + i
                                 : (static_cast<int64_t>(b) * p.Hq + h) * p.S + i;
}

// Row i of head h of sequence b in a strided bf16 tensor.
__device__ __forceinline__ const __nv_bfloat16* bwd_row(const __nv_bfloat16* base, const gptoss_strides& s, int b,
                                                        int64_t tok0, int i, int h, bool thd) {
  return thd ? base + (tok0 + i) * s.tok + static_cast<int64_t>(h) * s.head
             : base + static_cast<int64_t>(b) * s.batch + static_cast<int64_t>(i) * s.tok +
                   static_cast<int64_t>(h) * s.head;
}

__device__ __forceinline__ float dot8_bf16(const uint4& a, const uint4& b) {
  const uint32_t* x = reinterpret_cast<const uint32_t*>(&a);
  const uint32_t* y = reinterpret_cast<const uint32_t*>(&b);
  float acc = 0.f;
#pragma unroll
  for (int w = 0; w < 4; ++w) acc += bf16lo(x[w]) * bf16lo(y[w]) + bf16hi(x[w]) * bf16hi(y[w]);
  return acc;
}

// D = <dout, out> for 64 rows x every head of one sequence, and the sink
// gradient -sum_i exp(sink_h - lse_i) D_i of those rows.  Grid (tiles, B).
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(const __grid_constant__ BwdParams p) {
  __shared__ float part[kBwdMaxHeads];
  const int b = blockIdx.y;
  const BwdSeq sq = bwd_seq(p, b);
  const int i0 = blockIdx.x * kBwdTile;
  if (i0 >= sq.L) return;
  for (int h = threadIdx.x; h < p.Hq; h += blockDim.x) part[h] = 0.f;
  __syncthreads();
  const bool thd = p.cu_seqlens != nullptr;
  const int rows = min(kBwdTile, sq.L - i0);
  for (int it = threadIdx.x; it < rows * p.Hq; it += blockDim.x) {
    const int r = it / p.Hq, h = it - r * p.Hq;
    const int i = i0 + r;
    const uint4* o = reinterpret_cast<const uint4*>(bwd_row(p.out, p.so, b, sq.tok0, i, h, thd));
    const uint4* d = reinterpret_cast<const uint4*>(bwd_row(p.dout, p.sdo, b, sq.tok0, i, h, thd));
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc += dot8_bf16(__ldg(o + c), __ldg(d + c));
    const int64_t ri = bwd_row_index(p, b, h, i, sq.tok0);
    p.dsum[ri] = acc;
    const float lse = __ldg(p.lse + ri);
    p.lse2[ri] = lse * kLog2e;
    const float share = ex2_approx((__ldg(p.sinks + h) - lse) * kLog2e);
    atomicAdd(&part[h], -share * acc);
  }
  __syncthreads();
  for (int h = threadIdx.x; h < p.Hq; h += blockDim.x) atomicAdd(p.dsinks + h, part[h]);
}

// Is query row i allowed to see key j (both inside a sequence of length L)?
__device__ __forceinline__ bool bwd_visible(int i, int j, int L, int window) {
  return j <= i && i < L && (window == 0 || i - j < window);
}

// Rows (gr, gr + 8) of an mma.sync A fragment from global memory: 16 rows
// starting at row0 (stride `row_stride` elements between rows), invalid rows
// (>= n_valid) zero.
__device__ __forceinline__ void load_a_frag(uint32_t (&a)[4][4], const __nv_bfloat16* row_lo,
                                            const __nv_bfloat16* row_hi, bool lo_ok, bool hi_ok, int tq) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int c = kk * 16 + 2 * tq;
    a[kk][0] = lo_ok ? *reinterpret_cast<const uint32_t*>(row_lo + c) : 0u;
    a[kk][1] = hi_ok ? *reinterpret_cast<const uint32_t*>(row_hi + c) : 0u;
    a[kk][2] = lo_ok ? *reinterpret_cast<const uint32_t*>(row_lo + c + 8) : 0u;
    a[kk][3] = hi_ok ? *reinterpret_cast<const uint32_t*>(row_hi + c + 8) : 0u;
  }
}

// RoPE taken back (the adjoint c R(theta)^T of gpt_oss.rope_utils'
// apply_rotary_emb, R rotary pairs (j, j + R)): pair j's (x, y) = (g_j,
// g_{j+R}) -> (x cc + y cs, y cc - x cs) with (cc, cs) = the row's (c cos, c
// sin) of pair j; features past 2R pass through unchanged (they carry no
// concentration).
__device__ __forceinline__ void rope_t_pair(float x, float y, float2 c, float& xr, float& yr) {
  xr = x * c.x + y * c.y;
  yr = y * c.x - x * c.y;
}

// Writes a 16 x 64 fp32 accumulator (C fragments, rows gr / gr + 8) as bf16
// rows, optionally scaled and taken back through RoPE with R rotary pairs
// (rope_t_pair); a thread's features d = 8 nf + 2 tq + e and their partners
// d + R (fragment nf + R / 8) sit in the same thread.
template <int R>
__device__ __forceinline__ void store_rows(const float (&acc)[8][4], __nv_bfloat16* row_lo, __nv_bfloat16* row_hi,
                                           const float2* cs_lo, const float2* cs_hi, bool lo_ok, bool hi_ok,
                                           float scale, bool rotate, int tq) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const bool ok = half == 0 ? lo_ok : hi_ok;
    if (!ok) continue;
    __nv_bfloat16* row = half == 0 ? row_lo : row_hi;
    const float2* cs = half == 0 ? cs_lo : cs_hi;
    const int e0 = 2 * half;
    if (!rotate) {
#pragma unroll
      for (int nf = 0; nf < 8; ++nf)
        *reinterpret_cast<uint32_t*>(row + 8 * nf + 2 * tq) =
            pack_bf16(acc[nf][e0] * scale, acc[nf][e0 + 1] * scale);
      continue;
    }
    constexpr int kNp = R / 8;  // partner offset in fragments
#pragma unroll
    for (int nf = 0; nf < kNp; ++nf) {
      const int d = 8 * nf + 2 * tq;  // pairs d, d + 1 and their partners d + R, d + R + 1
      float xr[2], yr[2];
#pragma unroll
      for (int e = 0; e < 2; ++e)
        rope_t_pair(acc[nf][e0 + e] * scale, acc[nf + kNp][e0 + e] * scale, __ldg(cs + d + e), xr[e], yr[e]);
      *reinterpret_cast<uint32_t*>(row + d) = pack_bf16(xr[0], xr[1]);
      *reinterpret_cast<uint32_t*>(row + d + R) = pack_bf16(yr[0], yr[1]);
    }
#pragma unroll
    for (int nf = 2 * kNp; nf < 8; ++nf)  // past the rotary features
      *reinterpret_cast<uint32_t*>(row + 8 * nf + 2 * tq) =
          pack_bf16(acc[nf][e0] * scale, acc[nf][e0 + 1] * scale);
  }
}

// Split sweeps: dk = c R^T (scale dK_acc) and dv = dV_acc as bf16.  Thread
// (token, kv head, j) handles features j and j + 32.
__global__ void __launch_bounds__(256) attn_bwd_dkdv_finish_kernel(const __grid_constant__ BwdParams p) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(p.T) * p.Hkv * kPairs) return;
  const int j = static_cast<int>(idx % kPairs);
  const int64_t tg = idx / kPairs;  // token * Hkv + kv head
  const int64_t t = tg / p.Hkv;
  const int64_t row = tg * kHeadDim;
  // features j and j + 32: the rotary pair (j, j + R) is handled by its
  // first feature's thread, features past 2R pass through
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int f = j + u * kPairs;
    if (f < p.R) {
      float xr, yr;
      rope_t_pair(p.dk_acc[row + f] * p.scale, p.dk_acc[row + f + p.R] * p.scale, __ldg(p.cs + t * kPairs + f), xr,
                  yr);
      p.dk[row + f] = __float2bfloat16_rn(xr);
      p.dk[row + f + p.R] = __float2bfloat16_rn(yr);
    } else if (f >= 2 * p.R) {
      p.dk[row + f] = __float2bfloat16_rn(p.dk_acc[row + f] * p.scale);
    }
  }
  p.dv[row + j] = __float2bfloat16_rn(p.dv_acc[row + j]);
  p.dv[row + j + kPairs] = __float2bfloat16_rn(p.dv_acc[row + j + kPairs]);
}

struct __align__(128) BwdQSmem {
  uint8_t k[2][kBwdTile * 128];  // rotated k tile (fp16), 128B-swizzled rows
  uint8_t v[2][kBwdTile * 128];  // v tile (bf16)
};

// 3 CTAs per SM: at most 170 registers a thread.
// R: the call's rotary pairs (p.R), a template parameter so each
// instantiation holds one RoPE transpose (measured: a runtime switch among
// four cost the sliding-window backward 2.7 %).
template <int R>
__global__ void __launch_bounds__(kBwdThreads, 3) attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  __shared__ BwdQSmem sm;
  const int qt = p.n_tiles - 1 - static_cast<int>(blockIdx.x);  // the longest sweeps start first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / p.G;
  const BwdSeq sq = bwd_seq(p, b);
  const int i0 = qt * kBwdTile;
  if (i0 >= sq.L) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, tq = lane & 3;
  const bool thd = p.cu_seqlens != nullptr;
  const int L = sq.L, W = p.window;
  // key tiles this query tile sees
  const int j_first = W > 0 ? max(0, i0 - W + 1) : 0;
  const int kt_lo = j_first / kBwdTile, kt_hi = min(L - 1, i0 + kBwdTile - 1) / kBwdTile;
  const int n_it = kt_hi - kt_lo + 1;

  // this warp's 16 queries: rotated Q (fp16) and dout (bf16) as A fragments
  const int il = i0 + warp * 16 + gr, ih = il + 8;
  const bool il_ok = il < L, ih_ok = ih < L;
  uint32_t qa[4][4], da[4][4];
  load_a_frag(qa, p.qh + ((sq.tok0 + il) * p.Hq + h) * kHeadDim, p.qh + ((sq.tok0 + ih) * p.Hq + h) * kHeadDim,
              il_ok, ih_ok, tq);
  load_a_frag(da, bwd_row(p.dout, p.sdo, b, sq.tok0, il, h, thd), bwd_row(p.dout, p.sdo, b, sq.tok0, ih, h, thd),
              il_ok, ih_ok, tq);
  const float lse_l = il_ok ? __ldg(p.lse + bwd_row_index(p, b, h, il, sq.tok0)) * kLog2e : 0.f;
  const float lse_h = ih_ok ? __ldg(p.lse + bwd_row_index(p, b, h, ih, sq.tok0)) * kLog2e : 0.f;
  const float d_l = il_ok ? __ldg(p.dsum + bwd_row_index(p, b, h, il, sq.tok0)) : 0.f;
  const float d_h = ih_ok ? __ldg(p.dsum + bwd_row_index(p, b, h, ih, sq.tok0)) : 0.f;

  auto load = [&](int it, int buf) {
    const int j0 = (kt_lo + it) * kBwdTile;
    const uint32_t ks = smem_u32(sm.k[buf]), vs = smem_u32(sm.v[buf]);
    for (int c = tid; c < kBwdTile * 8; c += kBwdThreads) {
      const int r = c >> 3, ch = c & 7, j = j0 + r;
      if (j < L) {
        cp_async16(sw128_addr(ks, r, ch), p.kh + ((sq.tok0 + j) * p.Hkv + g) * kHeadDim + 8 * ch);
        cp_async16(sw128_addr(vs, r, ch), bwd_row(p.v, p.sv, b, sq.tok0, j, g, thd) + 8 * ch);
      } else {
        st_shared_zero16(sw128_addr(ks, r, ch));
        st_shared_zero16(sw128_addr(vs, r, ch));
      }
    }
  };

  float dq[8][4];
#pragma unroll
  for (int nf = 0; nf < 8; ++nf)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[nf][e] = 0.f;

  load(0, 0);
  cp_async_commit();
  for (int it = 0; it < n_it; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_it) {
      load(it + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j0 = (kt_lo + it) * kBwdTile;
    const uint32_t ks = smem_u32(sm.k[buf]), vs = smem_u32(sm.v[buf]);
    // S = Q K^T and dP = dout V^T: this warp's 16 queries x 64 keys
    float s[8][4], dpv[8][4];
#pragma unroll
    for (int nf = 0; nf < 8; ++nf) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nf][e] = dpv[nf][e] = 0.f;
      const int row = 8 * nf + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sw128_addr(ks, row, kp * 4 + (lane >> 3)), b0, b1, b2, b3);
        mma_f16_16816(s[nf], qa[2 * kp], b0, b1);
        mma_f16_16816(s[nf], qa[2 * kp + 1], b2, b3);
        ldsm_x4(sw128_addr(vs, row, kp * 4 + (lane >> 3)), b0, b1, b2, b3);
        mma_bf16_16816(dpv[nf], da[2 * kp], b0, b1);
        mma_bf16_16816(dpv[nf], da[2 * kp + 1], b2, b3);
      }
    }
    // dS = P (dP - D) on the visible pairs
#pragma unroll
    for (int nf = 0; nf < 8; ++nf)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = j0 + 8 * nf + 2 * tq + (e & 1);
        const int i = e < 2 ? il : ih;
        const bool vis = j < L && bwd_visible(i, j, L, W);
        const float pv = vis ? ex2_approx(s[nf][e] * p.scale_log2 - (e < 2 ? lse_l : lse_h)) : 0.f;
        dpv[nf][e] = pv * (dpv[nf][e] - (e < 2 ? d_l : d_h));
      }
    // dQ += dS K (contraction over the 64 keys)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t sa[4];
      sa[0] = pack_f16(dpv[2 * kk][0], dpv[2 * kk][1]);
      sa[1] = pack_f16(dpv[2 * kk][2], dpv[2 * kk][3]);
      sa[2] = pack_f16(dpv[2 * kk + 1][0], dpv[2 * kk + 1][1]);
      sa[3] = pack_f16(dpv[2 * kk + 1][2], dpv[2 * kk + 1][3]);
      const int row = 16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sw128_addr(ks, row, 2 * dp + (lane >> 4)), b0, b1, b2, b3);
        mma_f16_16816(dq[2 * dp], sa, b0, b1);
        mma_f16_16816(dq[2 * dp + 1], sa, b2, b3);
      }
    }
    __syncthreads();  // the buffer is refilled two iterations on
  }
  const int64_t tl = sq.tok0 + il, th = sq.tok0 + ih;
  __nv_bfloat16* rl = p.dq + (tl * p.Hq + h) * kHeadDim;
  __nv_bfloat16* rh = p.dq + (th * p.Hq + h) * kHeadDim;
  const float2 *cl = p.cs + tl * kPairs, *ch = p.cs + th * kPairs;
  store_rows<R>(dq, rl, rh, cl, ch, il_ok, ih_ok, p.scale, true, tq);
}

}  // namespace gptoss
