// bwd_host.cuh -- host side of the backward entry points of libgptoss_attn
// (declared in include/gptoss.h): gptoss_attn_bwd_workspace_size and
// gptoss_attn_bwd.  Included once by gptoss_lib.cu (one translation unit).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "gptoss.h"
#include "host_util.cuh"
#include "rope_qk.cuh"

using namespace gptoss;

namespace {

inline size_t bwd_round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: rotated q (fp16) | rotated k (fp16) | per-token (c cos, c sin)
// table | D = <dout, out> (fp32, lse layout) | lse log2(e) (fp32, lse layout)
// | dK and dV fp32 accumulators of split sweeps (adjacent, zeroed with one
// memset), each 256-byte aligned.
struct BwdWorkspace {
  size_t q, k, cs, d, l2, acc, acc_bytes, total;
};

inline BwdWorkspace bwd_workspace(int64_t T, int Hq, int Hkv) {
  BwdWorkspace w;
  w.q = 0;
  w.k = w.q + bwd_round256(static_cast<size_t>(T) * Hq * kHeadDim * 2);
  w.cs = w.k + bwd_round256(static_cast<size_t>(T) * Hkv * kHeadDim * 2);
  w.d = w.cs + bwd_round256(static_cast<size_t>(T) * kPairs * sizeof(float2));
  w.l2 = w.d + bwd_round256(static_cast<size_t>(T) * Hq * sizeof(float));
  w.acc = w.l2 + bwd_round256(static_cast<size_t>(T) * Hq * sizeof(float));
  w.acc_bytes = 2 * static_cast<size_t>(T) * Hkv * kHeadDim * sizeof(float);
  w.total = w.acc + bwd_round256(w.acc_bytes);
  return w;
}

}  // namespace

extern "C" {

size_t gptoss_attn_bwd_workspace_size(int32_t total_tokens, int32_t Hq, int32_t Hkv, int32_t D) {
  if (total_tokens <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D != kHeadDim) return 0;
  return bwd_workspace(total_tokens, Hq, Hkv).total;
}

gptoss_status gptoss_attn_bwd(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk, const void* v,
                              gptoss_strides sv, const void* out, gptoss_strides so, const void* dout,
                              gptoss_strides sdo, const float* lse, const float* sinks, const int32_t* positions,
                              const int32_t* cu_seqlens, int32_t B, int32_t S, int32_t total_tokens, int32_t Hq,
                              int32_t Hkv, int32_t D, int32_t window, float softmax_scale,
                              const gptoss_rope_params* rope, void* dq, void* dk, void* dv, float* dsinks,
                              void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  if (B < 0 || S < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || window < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (Hq > kBwdMaxHeads || B > 65535) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/true);
  if (st != GPTOSS_OK) return st;
  const bool thd = cu_seqlens != nullptr;
  if (!thd && static_cast<int64_t>(B) * S != total_tokens) return GPTOSS_ERR_INVALID_ARG;
  if (dsinks == nullptr) return GPTOSS_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (total_tokens == 0 || B == 0 || S == 0) {  // no rows: the sink gradient is zero
    return cudaMemsetAsync(dsinks, 0, sizeof(float) * Hq, s) == cudaSuccess ? GPTOSS_OK : GPTOSS_ERR_CUDA;
  }
  if (!q || !k || !v || !out || !dout || !lse || !sinks || !dq || !dk || !dv || !workspace)
    return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, !thd) || !strides_ok(sk, !thd) || !strides_ok(sv, !thd) || !strides_ok(so, !thd) ||
      !strides_ok(sdo, !thd))
    return GPTOSS_ERR_INVALID_ARG;
  const BwdWorkspace ws = bwd_workspace(total_tokens, Hq, Hkv);
  if (workspace_bytes < ws.total) return GPTOSS_ERR_INVALID_ARG;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);

  // 1. q and k rotated once (fp16) with every token's angle table; without
  //    RoPE the identity table (angle 0, concentration 1) converts them
  RopeQkParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.q = static_cast<const __nv_bfloat16*>(q);
  rp.k = static_cast<const __nv_bfloat16*>(k);
  rp.q_out = reinterpret_cast<__nv_bfloat16*>(wsb + ws.q);  // fp16 bits
  rp.k_out = reinterpret_cast<__nv_bfloat16*>(wsb + ws.k);
  rp.sq = sq;
  rp.sk = sk;
  rp.sqo.head = kHeadDim;
  rp.sqo.tok = static_cast<int64_t>(Hq) * kHeadDim;
  rp.sqo.batch = thd ? 0 : static_cast<int64_t>(S) * Hq * kHeadDim;
  rp.sko.head = kHeadDim;
  rp.sko.tok = static_cast<int64_t>(Hkv) * kHeadDim;
  rp.sko.batch = thd ? 0 : static_cast<int64_t>(S) * Hkv * kHeadDim;
  rp.tm.positions = positions;
  rp.tm.cu_seqlens = cu_seqlens;
  rp.tm.nseq = B;
  rp.tm.S = thd ? 0 : S;
  rp.tm.ntok = total_tokens;
  rp.Hq = Hq;
  rp.Hkv = Hkv;
  rp.D = kHeadDim;
  if (rope != nullptr) {
    yarn_table(*rope, &rp.tab);
  } else {
    memset(&rp.tab, 0, sizeof(rp.tab));  // every inverse frequency 0: cos 1, sin 0
    rp.tab.conc = 1.f;
    rp.tab.R = kPairs;
  }
  rp.cs_out = reinterpret_cast<float2*>(wsb + ws.cs);
  const int rgrid = (total_tokens + kRopeTokensPerCta - 1) / kRopeTokensPerCta;
  rope_qk_kernel<true><<<rgrid, kRopeThreads, 0, s>>>(rp);
  st = check_launch();
  if (st != GPTOSS_OK) return st;

  // 2. D = <dout, out> and the sink gradient
  if (cudaMemsetAsync(dsinks, 0, sizeof(float) * Hq, s) != cudaSuccess) return GPTOSS_ERR_CUDA;
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.qh = rp.q_out;
  p.kh = rp.k_out;
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.out = static_cast<const __nv_bfloat16*>(out);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.sv = sv;
  p.so = so;
  p.sdo = sdo;
  p.lse = lse;
  p.dsum = reinterpret_cast<float*>(wsb + ws.d);
  p.lse2 = reinterpret_cast<float*>(wsb + ws.l2);
  p.cs = rp.cs_out;
  p.R = rp.tab.R;
  p.sinks = sinks;
  p.dsinks = dsinks;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.S = S;
  p.T = total_tokens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.window = window;
  p.n_tiles = (S + kBwdTile - 1) / kBwdTile;
  p.scale = softmax_scale;
  p.scale_log2 = softmax_scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  // tensor maps of the tcgen05 kernels: (d, head, token, batch), 64-row
  // boxes; THD is one batch of total_tokens rows (its batch stride unused)
  {
    const uint64_t dimS = thd ? static_cast<uint64_t>(total_tokens) : static_cast<uint64_t>(S);
    const uint64_t dimB = thd ? 1 : static_cast<uint64_t>(B);
    const uint64_t kt_b = static_cast<uint64_t>(Hkv) * kHeadDim * 2, qt_b = static_cast<uint64_t>(Hq) * kHeadDim * 2;
    st = make_tmap_4d(&p.tmap_k, p.kh, kHeadDim, Hkv, dimS, dimB, kHeadDim * 2, kt_b, dimS * kt_b, kHeadDim, 1,
                      kBwdTcQ, 1, true);
    if (st != GPTOSS_OK) return st;
    st = make_tmap_4d(&p.tmap_q, p.qh, kHeadDim, Hq, dimS, dimB, kHeadDim * 2, qt_b, dimS * qt_b, kHeadDim, 1,
                      kBwdTcQ, 1, true);
    if (st != GPTOSS_OK) return st;
    const uint64_t vb = thd ? dimS * sv.tok * 2 : static_cast<uint64_t>(sv.batch) * 2;
    st = make_tmap_4d(&p.tmap_v, v, kHeadDim, Hkv, dimS, dimB, sv.head * 2, sv.tok * 2, vb == 0 ? 16 : vb,
                      kHeadDim, 1, kBwdTcQ, 1);
    if (st != GPTOSS_OK) return st;
    const uint64_t db = thd ? dimS * sdo.tok * 2 : static_cast<uint64_t>(sdo.batch) * 2;
    st = make_tmap_4d(&p.tmap_do, dout, kHeadDim, Hq, dimS, dimB, sdo.head * 2, sdo.tok * 2, db == 0 ? 16 : db,
                      kHeadDim, 1, kBwdTcQ, 1);
    if (st != GPTOSS_OK) return st;
  }
  // The longest dK / dV sweep (key tile 0 of the longest sequence): split it
  // into chunks of kBwdTcChunkIt steps when it has more, so no CTA runs far
  // longer than the rest; the chunks add into fp32 accumulators.
  const int64_t q_last0 = window > 0 ? std::min<int64_t>(S - 1, kBwdTcKeys - 1 + window - 1) : S - 1;
  const int64_t max_it = static_cast<int64_t>(p.G) * (q_last0 / kBwdTcQ + 1);
  const int64_t max_chunks = (max_it + kBwdTcChunkIt - 1) / kBwdTcChunkIt;
  const bool split = max_chunks > 1 && static_cast<int64_t>(B) * max_chunks <= 65535;
  p.max_chunks = split ? static_cast<int>(max_chunks) : 1;
  p.dk_acc = reinterpret_cast<float*>(wsb + ws.acc);
  p.dv_acc = p.dk_acc + static_cast<int64_t>(total_tokens) * Hkv * kHeadDim;
  if (split && cudaMemsetAsync(wsb + ws.acc, 0, ws.acc_bytes, s) != cudaSuccess) return GPTOSS_ERR_CUDA;
  attn_bwd_preprocess_kernel<<<dim3(p.n_tiles, B), 256, 0, s>>>(p);
  st = check_launch();
  if (st != GPTOSS_OK) return st;

  // 3. dK, dV (one CTA per key tile and kv head, or per chunk of its sweep)
  //    and 4. dQ (one per query tile and head)
  const int n_ktiles = (S + kBwdTcKeys - 1) / kBwdTcKeys;
  const size_t tc_smem = sizeof(BwdTcSmem) + 1024;
  auto dkdv = split ? attn_bwd_dkdv_tc_kernel<true> : attn_bwd_dkdv_tc_kernel<false>;
  if (cudaFuncSetAttribute(dkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(tc_smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  dkdv<<<dim3(n_ktiles, Hkv, B * p.max_chunks), kBwdTcThreads, tc_smem, s>>>(p);
  if (split) {
    st = check_launch();
    if (st != GPTOSS_OK) return st;
    const int64_t n = static_cast<int64_t>(total_tokens) * Hkv * kPairs;
    attn_bwd_dkdv_finish_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
  }
  st = check_launch();
  if (st != GPTOSS_OK) return st;
  // dQ: the tcgen05 kernel owns all tensor memory of its SM (one CTA at a
  // time), so its fixed cost per CTA -- allocation, first loads, filling and
  // draining the pipeline -- only pays off over long sweeps (full context or
  // windows of 1024+ keys: 16+ key tiles per query tile).  Short sweeps (a
  // 128-key window: 4-5 tiles) run faster on the mma.sync kernel, three
  // CTAs to an SM (measured, B=4 S=4096 W=128: 1.27 against 1.66 ms).
  // both dQ kernels are instantiated per rotary pair count (a multiple of 8
  // up to 32: check_rope admits rotary_dim in multiples of 16)
  if (window == 0 || window >= 1024) {
    void (*dq)(BwdParams) = p.R == 8    ? attn_bwd_dq_tc_kernel<8>
                            : p.R == 16 ? attn_bwd_dq_tc_kernel<16>
                            : p.R == 24 ? attn_bwd_dq_tc_kernel<24>
                                        : attn_bwd_dq_tc_kernel<32>;
    const size_t q_smem = sizeof(BwdTcQSmem) + 1024;
    if (cudaFuncSetAttribute(dq, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(q_smem)) !=
        cudaSuccess)
      return GPTOSS_ERR_CUDA;
    dq<<<dim3((S + 127) / 128, Hq, B), kBwdTcThreads, q_smem, s>>>(p);
  } else {
    void (*dq)(BwdParams) = p.R == 8    ? attn_bwd_dq_kernel<8>
                            : p.R == 16 ? attn_bwd_dq_kernel<16>
                            : p.R == 24 ? attn_bwd_dq_kernel<24>
                                        : attn_bwd_dq_kernel<32>;
    dq<<<dim3(p.n_tiles, Hq, B), kBwdThreads, 0, s>>>(p);
  }
  return check_launch();
}

}  // extern "C"
