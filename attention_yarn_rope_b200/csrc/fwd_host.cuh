// fwd_host.cuh -- host side of the RoPE and prefill entry points of
// libgptoss_attn (declared in include/gptoss.h): gptoss_rope_qk,
// gptoss_attn_fwd_workspace_size, gptoss_attn_fwd.  Included once by
// gptoss_lib.cu (the library is one translation unit).
#pragma once

#include <cuda_runtime.h>

#include "fwd128.cuh"
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
  if (D != kHeadDim && D != kMaxHeadDim) return GPTOSS_ERR_UNSUPPORTED;
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
  p.D = D;
  yarn_table(*rope, &p.tab);
  const int grid = static_cast<int>((ntok + kRopeTokensPerCta - 1) / kRopeTokensPerCta);
  rope_qk_kernel<false><<<grid, kRopeThreads, 0, as_stream(stream)>>>(p);
  return check_launch();
}

// Workspace of gptoss_attn_fwd: k (rotated) and v as fp16, each dense
// [token][Hkv][D] and rounded up to 256 bytes, then each token's D / 2
// (c cos, c sin) pairs ([token][D / 2] float2).
static size_t fwd_ws_kv_bytes(int32_t total_tokens, int32_t Hkv, int32_t D) {
  return (static_cast<size_t>(total_tokens) * Hkv * D * 2 + 255) & ~static_cast<size_t>(255);
}

size_t gptoss_attn_fwd_workspace_size(int32_t total_tokens, int32_t Hkv, int32_t D) {
  if (total_tokens < 0 || Hkv <= 0 || (D != kHeadDim && D != kMaxHeadDim)) return 0;
  return 2 * fwd_ws_kv_bytes(total_tokens, Hkv, D) + static_cast<size_t>(total_tokens) * (D / 2) * sizeof(float2);
}

// The identity rotation (every angle 0, concentration 1) of D / 2 pairs: the
// pre-pass and the rope warps then only convert bf16 to fp16, exactly.
static void identity_table(RopeTable* t, int D) {
  for (int j = 0; j < kMaxPairs; ++j) t->inv_freq[j] = 0.0;
  t->conc = 1.0f;
  t->enabled = 1;
  t->R = D / 2;
}

// One prefill call, validated: the self-attention entry point and the block
// form both launch through here.
struct PrefillCall {
  const void *q, *k, *v;
  gptoss_strides sq, sk, sv, so;
  const float* sinks;            // nullable in the block form
  const int32_t* positions;      // self-attention only
  const int32_t* cu_seqlens;     // self-attention only
  int32_t B, Sq, Sk, Tq, Tk;     // Sk / Tk: key rows per batch row / in all (self: equal to the query's)
  int32_t Hq, Hkv, D, window, delta;
  int32_t q_pos0, k_pos0;        // default positions of the first query / key row
  float scale;
  const gptoss_rope_params* rope;
  void* out;                     // bf16, strides so
  float* out_f32;                // block form (D = 64): dense fp32 [B, Sq, Hq, 64]
  float* lse;
  void* workspace;
  cudaStream_t stream;
};

static gptoss_status prefill_launch(const PrefillCall& c) {
  const bool thd = c.cu_seqlens != nullptr;
  const int n_qtiles = (c.Sq + kFwdTile - 1) / kFwdTile;
  const int G = c.Hq / c.Hkv;
  const bool d128 = c.D == kMaxHeadDim;
  const int HP = d128 ? G : (G + 1) / 2;  // units per kv group and query tile: single heads or head pairs
  const int64_t n_units = static_cast<int64_t>(n_qtiles) * c.B * c.Hkv * HP;
  if (n_units > INT32_MAX) return GPTOSS_ERR_UNSUPPORTED;
  // The register split inside the kernel assumes exactly its launch register
  // count per thread; anything else could stall the split.  Instantiations:
  // D = 64 or 128, with a sliding window or causal only.
  const auto kernel = d128 ? (c.window > 0 ? attn_fwd128_kernel<true> : attn_fwd128_kernel<false>)
                           : (c.window > 0 ? attn_fwd_kernel<true> : attn_fwd_kernel<false>);
  const int variant = (d128 ? 2 : 0) + (c.window > 0 ? 1 : 0);
  static int launch_regs[4] = {-1, -1, -1, -1};
  int& regs = launch_regs[variant];
  if (regs < 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return GPTOSS_ERR_CUDA;
    regs = fa.numRegs;
  }
  if (regs != (d128 ? kF128LaunchRegs : kFwdLaunchRegs)) return GPTOSS_ERR_UNSUPPORTED;
  int device = 0, n_sm = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  const int grid = static_cast<int>(n_units < n_sm ? n_units : n_sm);

  FwdParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t dimQ = thd ? static_cast<uint64_t>(c.Tq) : static_cast<uint64_t>(c.Sq);
  const uint64_t dimK = thd ? static_cast<uint64_t>(c.Tk) : static_cast<uint64_t>(c.Sk);
  const uint64_t dimB = thd ? 1 : static_cast<uint64_t>(c.B);
  const uint64_t qb_stride = thd ? dimQ * c.sq.tok * 2 : static_cast<uint64_t>(c.sq.batch) * 2;
  // boxes of 64 features (128 bytes, the swizzle span): a D = 128 row is two
  gptoss_status st = make_tmap_4d(&p.tmap_q, c.q, c.D, c.Hq, dimQ, dimB, c.sq.head * 2, c.sq.tok * 2,
                                  qb_stride == 0 ? 16 : qb_stride, kHeadDim, 1, kFwdTile, 1);
  if (st != GPTOSS_OK) return st;
  // fp16 k and v: dense [B, Sk, Hkv, D] / [T, Hkv, D] in the workspace
  uint8_t* ws = static_cast<uint8_t*>(c.workspace);
  const size_t kv_bytes = fwd_ws_kv_bytes(c.Tk, c.Hkv, c.D);
  const uint64_t tok_b = static_cast<uint64_t>(c.Hkv) * c.D * 2;
  const uint64_t seq_b = dimK * tok_b;
  st = make_tmap_4d(&p.tmap_k, ws, c.D, c.Hkv, dimK, dimB, c.D * 2, tok_b, seq_b, kHeadDim, 1, kFwdTile, 1, true);
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_v, ws + kv_bytes, c.D, c.Hkv, dimK, dimB, c.D * 2, tok_b, seq_b, kHeadDim, 1, kFwdTile,
                    1, true);
  if (st != GPTOSS_OK) return st;
  p.q = static_cast<const __nv_bfloat16*>(c.q);
  p.sq = c.sq;
  p.out = static_cast<__nv_bfloat16*>(c.out);
  p.so = c.so;
  p.out_f32 = c.out_f32;
  p.lse = c.lse;
  p.sinks = c.sinks;
  p.cu_seqlens = c.cu_seqlens;
  p.B = c.B;
  p.S = c.Sq;
  p.T = c.Tq;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.G = G;
  p.HP = HP;
  p.window = c.window;
  p.delta = c.delta;
  p.Lk = c.Sk;
  p.n_qtiles = n_qtiles;
  p.n_units = static_cast<int>(n_units);
  p.scale_log2 = c.scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  // positions feed RoPE only: without RoPE the kernels take the identity table
  if (c.rope != nullptr) yarn_table(*c.rope, &p.tab);
  else identity_table(&p.tab, c.D);
  p.positions = c.rope != nullptr ? c.positions : nullptr;
  // the first kernel: k rotated (at its positions) and v converted into the
  // workspace as fp16, and the per-token angle table of the query tokens
  const bool same_tokens = c.delta == 0 && c.Sk == c.Sq && c.q_pos0 == c.k_pos0;
  float2* q_table = reinterpret_cast<float2*>(ws + 2 * kv_bytes);
  RopeQkParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.k = static_cast<const __nv_bfloat16*>(c.k);
  rp.k_out = reinterpret_cast<__nv_bfloat16*>(ws);  // fp16 bits (rope_qk_kernel<true>)
  rp.sk = c.sk;
  rp.v = static_cast<const __nv_bfloat16*>(c.v);
  rp.v_out = reinterpret_cast<__nv_bfloat16*>(ws + kv_bytes);
  rp.sv = c.sv;
  rp.sko.head = rp.svo.head = c.D;
  rp.sko.tok = rp.svo.tok = static_cast<int64_t>(c.Hkv) * c.D;
  rp.sko.batch = rp.svo.batch = thd ? 0 : static_cast<int64_t>(c.Sk) * c.Hkv * c.D;
  rp.tm.positions = p.positions;
  rp.tm.cu_seqlens = c.cu_seqlens;
  rp.tm.nseq = c.B;
  rp.tm.S = thd ? 0 : c.Sk;
  rp.tm.ntok = c.Tk;
  rp.tm.pos_offset = c.k_pos0;
  rp.Hq = 0;
  rp.Hkv = c.Hkv;
  rp.D = c.D;
  rp.tab = p.tab;
  rp.cs_out = same_tokens ? q_table : nullptr;
  rope_qk_kernel<true><<<(c.Tk + kRopeTokensPerCta - 1) / kRopeTokensPerCta, kRopeThreads, 0, c.stream>>>(rp);
  st = check_launch();
  if (st != GPTOSS_OK) return st;
  if (!same_tokens) {  // the block form: the query tokens' angle table on its own
    RopeQkParams tp;
    memset(&tp, 0, sizeof(tp));
    tp.tm.nseq = c.B;
    tp.tm.S = c.Sq;
    tp.tm.ntok = c.Tq;
    tp.tm.pos_offset = c.q_pos0;
    tp.D = c.D;
    tp.tab = p.tab;
    tp.cs_out = q_table;
    rope_qk_kernel<true><<<(c.Tq + kRopeTokensPerCta - 1) / kRopeTokensPerCta, kRopeThreads, 0, c.stream>>>(tp);
    st = check_launch();
    if (st != GPTOSS_OK) return st;
  }
  p.cs_tab = q_table;
  const size_t smem = (d128 ? sizeof(Fwd128Smem) : sizeof(FwdSmem)) + 1024;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  kernel<<<grid, d128 ? kF128Threads : kFwdThreads, smem, c.stream>>>(p);
  return check_launch();
}

gptoss_status gptoss_attn_fwd(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk, const void* v,
                              gptoss_strides sv, const float* sinks, const int32_t* positions,
                              const int32_t* cu_seqlens, int32_t B, int32_t S, int32_t total_tokens, int32_t Hq,
                              int32_t Hkv, int32_t D, int32_t window, float softmax_scale,
                              const gptoss_rope_params* rope, void* out, gptoss_strides so, float* lse,
                              void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  if (B < 0 || S < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0 || window < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim && D != kMaxHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  // partial rotary is taken at D = 64; the D = 128 kernel rotates all 64 pairs
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/D == kHeadDim);
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
  PrefillCall c;
  memset(&c, 0, sizeof(c));
  c.q = q;
  c.k = k;
  c.v = v;
  c.sq = sq;
  c.sk = sk;
  c.sv = sv;
  c.so = so;
  c.sinks = sinks;
  c.positions = positions;
  c.cu_seqlens = cu_seqlens;
  c.B = B;
  c.Sq = c.Sk = S;
  c.Tq = c.Tk = total_tokens;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.D = D;
  c.window = window;
  c.scale = softmax_scale;
  c.rope = rope;
  c.out = out;
  c.lse = lse;
  c.workspace = workspace;
  c.stream = as_stream(stream);
  return prefill_launch(c);
}

size_t gptoss_attn_fwd_block_workspace_size(int32_t B, int32_t Sq, int32_t Sk, int32_t Hkv, int32_t D) {
  if (B < 0 || Sq < 0 || Sk < 0 || Hkv <= 0 || D != kHeadDim) return 0;
  const int64_t tq = static_cast<int64_t>(B) * Sq, tk = static_cast<int64_t>(B) * Sk;
  if (tq > INT32_MAX || tk > INT32_MAX) return 0;
  return 2 * fwd_ws_kv_bytes(static_cast<int32_t>(tk), Hkv, kHeadDim) + static_cast<size_t>(tq) * kPairs * sizeof(float2);
}

gptoss_status gptoss_attn_fwd_block(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk,
                                    const void* v, gptoss_strides sv, int32_t B, int32_t Sq, int32_t Sk,
                                    int32_t q_start, int32_t k_start, int32_t Hq, int32_t Hkv, int32_t D,
                                    float softmax_scale, const gptoss_rope_params* rope, float* out, float* lse,
                                    void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  if (B < 0 || Sq < 0 || Sk < 0 || Hq <= 0 || Hkv <= 0 || q_start < 0 || k_start < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  // the key block must start at or before the query shard (causal: a block
  // after it is invisible), so every query row sees at least one key
  if (k_start > q_start) return GPTOSS_ERR_INVALID_ARG;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/true);
  if (st != GPTOSS_OK) return st;
  if (B == 0 || Sq == 0) return GPTOSS_OK;
  if (Sk == 0) return GPTOSS_ERR_INVALID_ARG;
  if (static_cast<int64_t>(q_start) + Sq > INT32_MAX || static_cast<int64_t>(q_start) - k_start > INT32_MAX)
    return GPTOSS_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !lse) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, true) || !strides_ok(sk, true) || !strides_ok(sv, true)) return GPTOSS_ERR_INVALID_ARG;
  const size_t need = gptoss_attn_fwd_block_workspace_size(B, Sq, Sk, Hkv, D);
  if (need == 0 || workspace == nullptr || !aligned16(workspace) || workspace_bytes < need)
    return GPTOSS_ERR_INVALID_ARG;
  PrefillCall c;
  memset(&c, 0, sizeof(c));
  c.q = q;
  c.k = k;
  c.v = v;
  c.sq = sq;
  c.sk = sk;
  c.sv = sv;
  c.B = B;
  c.Sq = Sq;
  c.Sk = Sk;
  c.Tq = B * Sq;
  c.Tk = B * Sk;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.D = kHeadDim;
  c.window = 0;
  c.delta = q_start - k_start;
  c.q_pos0 = q_start;
  c.k_pos0 = k_start;
  c.scale = softmax_scale;
  c.rope = rope;
  c.out_f32 = out;
  c.lse = lse;
  c.workspace = workspace;
  c.stream = as_stream(stream);
  return prefill_launch(c);
}

}  // extern "C"
