// qkv_rope.cuh -- the q, k, v projections of the attention input with RoPE
// in the GEMM epilogue (gptoss_qkv_rope).
//
// Rule: GptOssAttention's q_proj / k_proj / v_proj are Linear layers with
// bias (blog page "gpt-oss-20b 模型结构": 2880 -> 4096 / 512 / 512), y = x W^T
// + b; q and k, viewed as [token, head, head_dim], are then rotated by the
// YaRN RoPE of the gpt_oss.rope_utils page (apply_rotary_emb_qk: half-split
// pairs (j, j + D/2), concentration applied).  The three weights arrive
// stacked row-wise (q rows, k rows, v rows), the biases likewise.
//
// Design: one persistent GEMM over the stacked output features, tensor-core
// bound (x W^T is a dense contraction: 2 x 2880 FLOP per output).  Tiles of
// 128 tokens x 256 output features (measured: 1.0 PFLOP/s with 128 x 128
// tiles, whose operands cross L2 twice as often per FLOP), K in steps of 64
// (128 bytes of bf16, one swizzle span).  Warp 0 streams the x and W tiles
// with TMA through a ring of stages; warp 1 issues tcgen05.mma (M128 N256
// K16, bf16 -> fp32 in tensor memory) into one of two 256-column
// accumulators; warps 2-5 drain the other accumulator meanwhile -- each
// thread one token row: the tile's 256 / D heads, each wholly inside q, k or
// v, bias added, q and k heads rotated with the token's angles (a per-token
// table written by the first kernel of the call), rounded to bf16 and
// stored.
#pragma once

#include "host_util.cuh"
#include "rope_qk.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

constexpr int kPjBM = 128, kPjBN = 256, kPjBK = 64;
constexpr int kPjStages = 4;
constexpr int kPjThreads = 192;                  // producer, MMA issuer, 4 epilogue warps
constexpr int kPjABytes = kPjBM * kPjBK * 2;     // 16 KB of x per stage
constexpr int kPjBBytes = kPjBN * kPjBK * 2;     // 32 KB of W per stage
constexpr uint32_t kPjTmemCols = 512;            // two 256-column accumulators

struct ProjParams {
  CUtensorMap tmap_x;  // x: dims (hidden, T), box (64, 128)
  CUtensorMap tmap_w;  // stacked W: dims (hidden, N), box (64, 256)
  const __nv_bfloat16* bias;  // [N] nullable
  const float2* cs;           // [T][D / 2] (c cos, c sin), nullable: no rotation
  __nv_bfloat16 *q, *k, *v;
  gptoss_strides sq, sk, sv;  // token t of batch row b = t / S (BSHD) or t (THD, S = 0)
  int T, S, N, Hq, Hkv, n_ntiles, n_tiles, n_ksteps;
  uint64_t wait_ns;
};

struct __align__(1024) ProjSmem {
  uint8_t a[kPjStages][kPjABytes];
  uint8_t b[kPjStages][kPjBBytes];
  uint64_t full[kPjStages], empty[kPjStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

__device__ __forceinline__ void proj_producer(const ProjParams& p, ProjSmem& sm) {
  tma_prefetch_desc(&p.tmap_x);
  tma_prefetch_desc(&p.tmap_w);
  uint32_t it = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const int m0 = (tile / p.n_ntiles) * kPjBM, n0 = (tile % p.n_ntiles) * kPjBN;
    for (int ks = 0; ks < p.n_ksteps; ++ks, ++it) {
      const int s = it % kPjStages;
      if (!mbar_wait(&sm.empty[s], ((it / kPjStages) & 1) ^ 1, p.wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.full[s], kPjABytes + kPjBBytes);
      tma_load_4d(sm.a[s], &p.tmap_x, &sm.full[s], ks * kPjBK, m0, 0, 0);
      tma_load_4d(sm.b[s], &p.tmap_w, &sm.full[s], ks * kPjBK, n0, 0, 0);
    }
  }
  // the copies of the last stages must land before the CTA exits
  for (uint32_t i = it > kPjStages ? it - kPjStages : 0; i < it; ++i)
    mbar_wait(&sm.full[i % kPjStages], (i / kPjStages) & 1, p.wait_ns);
}

__device__ __forceinline__ void proj_mma(const ProjParams& p, ProjSmem& sm, uint32_t tmem) {
  constexpr uint32_t idesc = idesc_bf16_f32(kPjBM, kPjBN, false);  // x and W both K-major
  uint32_t it = 0, tc = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, ++tc) {
    const uint32_t buf = tc & 1;
    // the epilogue has drained this accumulator's previous tile
    if (tc >= 2 && !mbar_wait(&sm.acc_empty[buf], ((tc >> 1) - 1) & 1, p.wait_ns)) break;
    tc_fence_after();
    const uint32_t acc = tmem + buf * kPjBN;
    for (int ks = 0; ks < p.n_ksteps; ++ks, ++it) {
      const int s = it % kPjStages;
      if (!mbar_wait(&sm.full[s], (it / kPjStages) & 1, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      const uint64_t ad = sw128_desc(smem_u32(sm.a[s]));
      const uint64_t bd = sw128_desc(smem_u32(sm.b[s]));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(acc, ad + static_cast<uint64_t>(kk * 2), bd + static_cast<uint64_t>(kk * 2), idesc,
               (ks | kk) > 0 ? 1u : 0u);
      mma_commit(&sm.empty[s]);  // the stage is free once these products have read it
    }
    if (!ok) break;
    mma_commit(&sm.acc_full[buf]);
  }
}

// One token row of a tile: kD-feature heads, bias, RoPE on q / k, bf16 out.
template <int kD>
__device__ __forceinline__ void proj_epilogue(const ProjParams& p, ProjSmem& sm, uint32_t tmem) {
  const int wq = (threadIdx.x >> 5) & 3;  // TMEM lane quarter of this warp (warps 2-5 cover all four)
  const int r = wq * 32 + (threadIdx.x & 31);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  constexpr int kR = kD / 2;
  uint32_t tc = 0;
  for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++tc) {
    const uint32_t buf = tc & 1;
    if (!mbar_wait_warp(&sm.acc_full[buf], (tc >> 1) & 1, p.wait_ns)) return;
    tc_fence_after();
    const int m0 = (tile / p.n_ntiles) * kPjBM, n0 = (tile % p.n_ntiles) * kPjBN;
    const int t = m0 + r;
#pragma unroll 1
    for (int hh = 0; hh < kPjBN / kD; ++hh) {
      uint32_t a[kD];
#pragma unroll
      for (int c = 0; c < kD / 32; ++c)
        tmem_ld32(lane_base + buf * kPjBN + hh * kD + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32 * c]));
      tmem_wait_ld();
      const int col = n0 + hh * kD;  // first output feature of this head
      // a row past the tokens (zero-filled x) or a head past N (zero-filled W) stores nothing
      if (t < p.T && col < p.N) {
        float y[kD];
        if (p.bias != nullptr) {
          const uint4* bb = reinterpret_cast<const uint4*>(p.bias + col);
#pragma unroll
          for (int e = 0; e < kD / 8; ++e) {
            const uint4 w = __ldg(bb + e);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              y[8 * e + 2 * u] = __uint_as_float(a[8 * e + 2 * u]) + bf16lo(ww[u]);
              y[8 * e + 2 * u + 1] = __uint_as_float(a[8 * e + 2 * u + 1]) + bf16hi(ww[u]);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < kD; ++e) y[e] = __uint_as_float(a[e]);
        }
        const int qcols = p.Hq * kD, kcols = p.Hkv * kD;
        __nv_bfloat16* dst;
        const int64_t bi = p.S > 0 ? t / p.S : 0, si = p.S > 0 ? t % p.S : t;
        if (col < qcols) {
          dst = p.q + bi * p.sq.batch + si * p.sq.tok + static_cast<int64_t>(col / kD) * p.sq.head;
        } else if (col < qcols + kcols) {
          dst = p.k + bi * p.sk.batch + si * p.sk.tok + static_cast<int64_t>((col - qcols) / kD) * p.sk.head;
        } else {
          dst = p.v + bi * p.sv.batch + si * p.sv.tok + static_cast<int64_t>((col - qcols - kcols) / kD) * p.sv.head;
        }
        if (p.cs != nullptr && col < qcols + kcols) {  // q or k: pairs (j, j + D/2)
          const float4* cs = reinterpret_cast<const float4*>(p.cs + static_cast<int64_t>(t) * kR);
#pragma unroll
          for (int j2 = 0; j2 < kR / 2; ++j2) {
            const float4 c = __ldg(cs + j2);
            const int j = 2 * j2;
            const float x0 = y[j], x1 = y[j + 1], z0 = y[j + kR], z1 = y[j + kR + 1];
            y[j] = x0 * c.x - z0 * c.y;
            y[j + kR] = z0 * c.x + x0 * c.y;
            y[j + 1] = x1 * c.z - z1 * c.w;
            y[j + kR + 1] = z1 * c.z + x1 * c.w;
          }
        }
#pragma unroll
        for (int e = 0; e < kD / 8; ++e) {
          uint4 o;
          o.x = pack_bf16(y[8 * e], y[8 * e + 1]);
          o.y = pack_bf16(y[8 * e + 2], y[8 * e + 3]);
          o.z = pack_bf16(y[8 * e + 4], y[8 * e + 5]);
          o.w = pack_bf16(y[8 * e + 6], y[8 * e + 7]);
          reinterpret_cast<uint4*>(dst)[e] = o;
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&sm.acc_empty[buf]);
  }
}

template <int kD>
__global__ void __launch_bounds__(kPjThreads, 1) qkv_rope_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  ProjSmem& sm = *reinterpret_cast<ProjSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], 128);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kPjTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp == 0) {
    if (lane == 0) proj_producer(p, sm);
  } else if (warp == 1) {
    if (lane == 0) proj_mma(p, sm, tmem);
  } else {
    proj_epilogue<kD>(p, sm, tmem);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPjTmemCols);
  }
}

}  // namespace gptoss

extern "C" {

size_t gptoss_qkv_rope_workspace_size(int32_t total_tokens, int32_t D) {
  using namespace gptoss;
  if (total_tokens < 0 || (D != kHeadDim && D != kMaxHeadDim)) return 0;
  return static_cast<size_t>(total_tokens) * (D / 2) * sizeof(float2) + 16;
}

gptoss_status gptoss_qkv_rope(const void* x, int64_t x_row_stride, const void* w_qkv, const void* b_qkv,
                              const int32_t* positions, const int32_t* cu_seqlens, int32_t B, int32_t S_or_T,
                              int32_t hidden, int32_t Hq, int32_t Hkv, int32_t D, const gptoss_rope_params* rope,
                              void* q_out, gptoss_strides sq, void* k_out, gptoss_strides sk, void* v_out,
                              gptoss_strides sv, void* workspace, size_t workspace_bytes,
                              struct CUstream_st* stream) {
  using namespace gptoss;
  if (B < 0 || S_or_T < 0 || hidden <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim && D != kMaxHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  // whole 16-byte rows of x
  if (hidden % 8) return GPTOSS_ERR_UNSUPPORTED;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/false);
  if (st != GPTOSS_OK) return st;
  const bool thd = cu_seqlens != nullptr;
  const int64_t T = thd ? S_or_T : static_cast<int64_t>(B) * S_or_T;
  if (T == 0 || B == 0) return GPTOSS_OK;
  if (T > INT32_MAX) return GPTOSS_ERR_INVALID_ARG;
  if (!x || !w_qkv || !q_out || !k_out || !v_out) return GPTOSS_ERR_INVALID_ARG;
  if (x_row_stride < hidden || (x_row_stride * 2) % 16 != 0) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(v_out) ||
      (b_qkv != nullptr && !aligned16(b_qkv)))
    return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, !thd) || !strides_ok(sk, !thd) || !strides_ok(sv, !thd)) return GPTOSS_ERR_INVALID_ARG;
  if (rope != nullptr && (workspace == nullptr || !aligned16(workspace) ||
                          workspace_bytes < gptoss_qkv_rope_workspace_size(static_cast<int32_t>(T), D)))
    return GPTOSS_ERR_INVALID_ARG;
  const cudaStream_t s = as_stream(stream);
  ProjParams p;
  memset(&p, 0, sizeof(p));
  const int N = (Hq + 2 * Hkv) * D;
  st = make_tmap_4d(&p.tmap_x, x, hidden, T, 1, 1, x_row_stride * 2, x_row_stride * 2 * T, x_row_stride * 2 * T,
                    kPjBK, kPjBM, 1, 1);
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_w, w_qkv, hidden, N, 1, 1, static_cast<uint64_t>(hidden) * 2,
                    static_cast<uint64_t>(hidden) * 2 * N, static_cast<uint64_t>(hidden) * 2 * N, kPjBK, kPjBN, 1, 1);
  if (st != GPTOSS_OK) return st;
  p.bias = static_cast<const __nv_bfloat16*>(b_qkv);
  p.q = static_cast<__nv_bfloat16*>(q_out);
  p.k = static_cast<__nv_bfloat16*>(k_out);
  p.v = static_cast<__nv_bfloat16*>(v_out);
  p.sq = sq;
  p.sk = sk;
  p.sv = sv;
  p.T = static_cast<int>(T);
  p.S = thd ? 0 : S_or_T;
  p.N = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  const int n_mtiles = static_cast<int>((T + kPjBM - 1) / kPjBM);
  p.n_ntiles = (N + kPjBN - 1) / kPjBN;
  p.n_tiles = n_mtiles * p.n_ntiles;
  p.n_ksteps = (hidden + kPjBK - 1) / kPjBK;
  p.wait_ns = wait_limit_ns();
  if (rope != nullptr) {  // the first kernel: every token's angles, [T][D / 2]
    RopeQkParams tp;
    memset(&tp, 0, sizeof(tp));
    tp.tm.positions = positions;
    tp.tm.cu_seqlens = cu_seqlens;
    tp.tm.nseq = B;
    tp.tm.S = thd ? 0 : S_or_T;
    tp.tm.ntok = static_cast<int>(T);
    tp.D = D;
    yarn_table(*rope, &tp.tab);
    tp.cs_out = static_cast<float2*>(workspace);
    rope_qk_kernel<false><<<static_cast<unsigned>((T + kRopeTokensPerCta - 1) / kRopeTokensPerCta), kRopeThreads,
                            0, s>>>(tp);
    st = check_launch();
    if (st != GPTOSS_OK) return st;
    p.cs = static_cast<const float2*>(workspace);
  }
  int device = 0, n_sm = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  const int grid = p.n_tiles < n_sm ? p.n_tiles : n_sm;
  const size_t smem = sizeof(ProjSmem) + 1024;
  const auto kernel = D == kHeadDim ? qkv_rope_kernel<kHeadDim> : qkv_rope_kernel<kMaxHeadDim>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  kernel<<<grid, kPjThreads, smem, s>>>(p);
  return check_launch();
}

}  // extern "C"
