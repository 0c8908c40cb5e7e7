// fwd_host.cuh -- host side of the RoPE and prefill entry points of
// libgptoss_attn (declared in include/gptoss.h): gptoss_rope_qk,
// gptoss_attn_fwd_workspace_size, gptoss_attn_fwd.  Included once by
// gptoss_lib.cu (the library is one translation unit).
#pragma once

#include <cuda_runtime.h>

#include "fwd_pipeline.cuh"
#include "gptoss.h"
#include "host_util.cuh"
#include "rope_qk.cuh"

using namespace gptoss;

extern "C" {

gptoss_status gptoss_rope_qk(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk, void* q_out,
                             gptoss_strides sq_out, void* k_out, gptoss_strides sk_out, const int32_t* positions,
                             const int32_t* cu_seqlens, int32_t B, int32_t S_or_T, int32_t Hq, int32_t Hkv,
                             int32_t D, const gptoss_rope_params* rope, struct CUstream_st* stream) {
  if (rope == nullptr) return GPTOSS_ERR_INVALID_ARG;
  if (B < 0 || S_or_T < 0 || Hq <= 0 || Hkv <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/true);
  if (st != GPTOSS_OK) return st;
  const bool thd = cu_seqlens != nullptr;
  const int64_t ntok = thd ? S_or_T : static_cast<int64_t>(B) * S_or_T;
  if (ntok == 0 || B == 0) return GPTOSS_OK;
  if (ntok > INT32_MAX) return GPTOSS_ERR_INVALID_ARG;
  if (!q || !k || !q_out || !k_out) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out)) return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, !thd) || !strides_ok(sk, !thd) || !strides_ok(sq_out, !thd) || !strides_ok(sk_out, !thd))
    return GPTOSS_ERR_INVALID_ARG;
  RopeQkParams p;
  memset(&p, 0, sizeof(p));  // no angle table output (cs_out = nullptr)
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.k_out = static_cast<__nv_bfloat16*>(k_out);
  p.sq = sq;
  p.sk = sk;
  p.sqo = sq_out;
  p.sko = sk_out;
  p.tm.positions = positions;
  p.tm.cu_seqlens = cu_seqlens;
  p.tm.nseq = B;
  p.tm.S = thd ? 0 : S_or_T;
  p.tm.ntok = static_cast<int>(ntok);
  p.Hq = Hq;
  p.Hkv = Hkv;
  yarn_table(*rope, &p.tab);
  const int grid = static_cast<int>((ntok + kRopeTokensPerCta - 1) / kRopeTokensPerCta);
  rope_qk_kernel<false><<<grid, kRopeThreads, 0, as_stream(stream)>>>(p);
  return check_launch();
}

// Workspace of gptoss_attn_fwd: k (rotated) and v as fp16, each dense
// [token][Hkv][64] and rounded up to 256 bytes, then each token's 32
// (c cos, c sin) pairs ([token][32] float2).
static size_t fwd_ws_kv_bytes(int32_t total_tokens, int32_t Hkv) {
  return (static_cast<size_t>(total_tokens) * Hkv * kHeadDim * 2 + 255) & ~static_cast<size_t>(255);
}

size_t gptoss_attn_fwd_workspace_size(int32_t total_tokens, int32_t Hkv, int32_t D) {
  if (total_tokens < 0 || Hkv <= 0 || D != kHeadDim) return 0;
  return 2 * fwd_ws_kv_bytes(total_tokens, Hkv) + static_cast<size_t>(total_tokens) * kPairs * sizeof(float2);
}

// The identity rotation (every angle 0, concentration 1): the pre-pass and
// the rope warps then only convert bf16 to fp16, exactly.
static void identity_table(RopeTable* t) {
  for (int j = 0; j < kPairs; ++j) t->inv_freq[j] = 0.0;
  t->conc = 1.0f;
  t->enabled = 1;
  t->R = kPairs;
}

gptoss_status gptoss_attn_fwd(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk, const void* v,
                              gptoss_strides sv, const float* sinks, const int32_t* positions,
                              const int32_t* cu_seqlens, int32_t B, int32_t S, int32_t total_tokens, int32_t Hq,
                              int32_t Hkv, int32_t D, int32_t window, float softmax_scale,
                              const gptoss_rope_params* rope, void* out, gptoss_strides so, float* lse,
                              void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  if (B < 0 || S < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || window < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/true);
  if (st != GPTOSS_OK) return st;
  const bool thd = cu_seqlens != nullptr;
  if (!thd && static_cast<int64_t>(B) * S != total_tokens) return GPTOSS_ERR_INVALID_ARG;
  if (total_tokens == 0 || B == 0 || S == 0) return GPTOSS_OK;
  if (!q || !k || !v || !sinks || !out) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, !thd) || !strides_ok(sk, !thd) || !strides_ok(sv, !thd) || !strides_ok(so, !thd))
    return GPTOSS_ERR_INVALID_ARG;
  // k (rotated) and v are written once into the workspace as fp16, the
  // operand format of both products
  if (workspace == nullptr || !aligned16(workspace) ||
      workspace_bytes < gptoss_attn_fwd_workspace_size(total_tokens, Hkv, D))
    return GPTOSS_ERR_INVALID_ARG;
  const int n_qtiles = (S + kFwdTile - 1) / kFwdTile;
  const int G = Hq / Hkv;
  const int HP = (G + 1) / 2;  // head pairs per kv group
  const int64_t n_units = static_cast<int64_t>(n_qtiles) * B * Hkv * HP;
  if (n_units > INT32_MAX) return GPTOSS_ERR_UNSUPPORTED;
  // The register split inside the kernel assumes exactly kFwdLaunchRegs
  // registers per thread at launch; anything else could stall the split.
  static int launch_regs = -1;
  if (launch_regs < 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_fwd_kernel) != cudaSuccess) return GPTOSS_ERR_CUDA;
    launch_regs = fa.numRegs;
  }
  if (launch_regs != kFwdLaunchRegs) return GPTOSS_ERR_UNSUPPORTED;
  int device = 0, n_sm = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  const int grid = static_cast<int>(n_units < n_sm ? n_units : n_sm);

  FwdParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t dimS = thd ? static_cast<uint64_t>(total_tokens) : static_cast<uint64_t>(S);
  const uint64_t dimB = thd ? 1 : static_cast<uint64_t>(B);
  const uint64_t qb_stride = thd ? dimS * sq.tok * 2 : static_cast<uint64_t>(sq.batch) * 2;
  st = make_tmap_4d(&p.tmap_q, q, kHeadDim, Hq, dimS, dimB, sq.head * 2, sq.tok * 2,
                         qb_stride == 0 ? 16 : qb_stride, kHeadDim, 1, kFwdTile, 1);
  if (st != GPTOSS_OK) return st;
  // fp16 k and v: dense [B, S, Hkv, D] / [T, Hkv, D] in the workspace
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t kv_bytes = fwd_ws_kv_bytes(total_tokens, Hkv);
  const uint64_t tok_b = static_cast<uint64_t>(Hkv) * kHeadDim * 2;
  const uint64_t seq_b = thd ? dimS * tok_b : static_cast<uint64_t>(S) * tok_b;
  st = make_tmap_4d(&p.tmap_k, ws, kHeadDim, Hkv, dimS, dimB, kHeadDim * 2, tok_b, seq_b, kHeadDim, 1, kFwdTile, 1,
                    true);
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_v, ws + kv_bytes, kHeadDim, Hkv, dimS, dimB, kHeadDim * 2, tok_b, seq_b, kHeadDim, 1,
                    kFwdTile, 1, true);
  if (st != GPTOSS_OK) return st;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.sq = sq;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.so = so;
  p.lse = lse;
  p.sinks = sinks;
  p.positions = positions;
  p.cu_seqlens = cu_seqlens;
  p.B = B;
  p.S = S;
  p.T = total_tokens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.HP = HP;
  p.window = window;
  p.n_qtiles = n_qtiles;
  p.n_units = static_cast<int>(n_units);
  p.scale_log2 = softmax_scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  // positions feed RoPE only: without RoPE the kernels take the identity table
  if (rope != nullptr) yarn_table(*rope, &p.tab);
  else identity_table(&p.tab);
  p.positions = rope != nullptr ? positions : nullptr;
  RopeQkParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.k = static_cast<const __nv_bfloat16*>(k);
  rp.k_out = reinterpret_cast<__nv_bfloat16*>(ws);  // fp16 bits (rope_qk_kernel<true>)
  rp.sk = sk;
  rp.v = static_cast<const __nv_bfloat16*>(v);
  rp.v_out = reinterpret_cast<__nv_bfloat16*>(ws + kv_bytes);
  rp.sv = sv;
  rp.sko.head = rp.svo.head = kHeadDim;
  rp.sko.tok = rp.svo.tok = static_cast<int64_t>(Hkv) * kHeadDim;
  rp.sko.batch = rp.svo.batch = thd ? 0 : static_cast<int64_t>(S) * Hkv * kHeadDim;
  rp.tm.positions = p.positions;
  rp.tm.cu_seqlens = cu_seqlens;
  rp.tm.nseq = B;
  rp.tm.S = thd ? 0 : S;
  rp.tm.ntok = total_tokens;
  rp.Hq = 0;
  rp.Hkv = Hkv;
  rp.tab = p.tab;
  rp.cs_out = reinterpret_cast<float2*>(ws + 2 * kv_bytes);
  p.cs_tab = rp.cs_out;
  const int rgrid = (total_tokens + kRopeTokensPerCta - 1) / kRopeTokensPerCta;
  rope_qk_kernel<true><<<rgrid, kRopeThreads, 0, as_stream(stream)>>>(rp);
  st = check_launch();
  if (st != GPTOSS_OK) return st;
  const size_t smem = sizeof(FwdSmem) + 1024;
  if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  attn_fwd_kernel<<<grid, kFwdThreads, smem, as_stream(stream)>>>(p);
  return check_launch();
}

}  // extern "C"
