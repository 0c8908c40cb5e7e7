// gptoss_lib.cu -- the C ABI of libgptoss_attn (declared in include/gptoss.h).
// One translation unit: the kernels live in the headers included below.
// Every entry point validates on the host, encodes its TMA descriptors and
// launches asynchronously on the caller's stream; nothing is allocated.

#include <cuda_runtime.h>

#include <mutex>

#include "attn_decode.cuh"
#include "fwd_pipeline.cuh"
#include "gptoss.h"
#include "host_util.cuh"
#include "rope_qk.cuh"
#include "sm100_ptx.cuh"

using namespace gptoss;

namespace {

// One mbarrier that nothing ever arrives at: the kernel's bounded wait must
// give up and record GPTOSS_ERR_TIMEOUT.  Exercises the device failure path.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns, int* result) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0, limit_ns);
  if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

}  // namespace

extern "C" {

const char* gptoss_status_string(gptoss_status s) {
  switch (s) {
    case GPTOSS_OK: return "GPTOSS_OK";
    case GPTOSS_ERR_INVALID_ARG: return "GPTOSS_ERR_INVALID_ARG";
    case GPTOSS_ERR_UNSUPPORTED: return "GPTOSS_ERR_UNSUPPORTED";
    case GPTOSS_ERR_CUDA: return "GPTOSS_ERR_CUDA";
    case GPTOSS_ERR_TIMEOUT: return "GPTOSS_ERR_TIMEOUT";
  }
  return "GPTOSS_ERR_UNKNOWN";
}

gptoss_status gptoss_set_wait_limit(uint32_t microseconds) {
  wait_limit_ns() = microseconds == 0 ? 2000000000ull : static_cast<uint64_t>(microseconds) * 1000ull;
  return GPTOSS_OK;
}

gptoss_status gptoss_read_device_status(int32_t* status_out, int32_t reset, struct CUstream_st* stream) {
  if (status_out == nullptr) return GPTOSS_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  if (reset) {
    static const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return GPTOSS_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return GPTOSS_ERR_CUDA;
  *status_out = v;
  return GPTOSS_OK;
}

gptoss_status gptoss_selftest_wait_timeout(uint32_t limit_us, int32_t* result_dev, struct CUstream_st* stream) {
  if (result_dev == nullptr || limit_us == 0 || limit_us > 1000000) return GPTOSS_ERR_INVALID_ARG;
  wait_timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_us) * 1000ull,
                                                             reinterpret_cast<int*>(result_dev));
  return check_launch();
}

gptoss_status gptoss_rope_qk(const void* q, gptoss_strides sq, const void* k, gptoss_strides sk, void* q_out,
                             gptoss_strides sq_out, void* k_out, gptoss_strides sk_out, const int32_t* positions,
                             const int32_t* cu_seqlens, int32_t B, int32_t S_or_T, int32_t Hq, int32_t Hkv,
                             int32_t D, const gptoss_rope_params* rope, struct CUstream_st* stream) {
  if (rope == nullptr) return GPTOSS_ERR_INVALID_ARG;
  if (B < 0 || S_or_T < 0 || Hq <= 0 || Hkv <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  gptoss_status st = check_rope(rope, D);
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

// Workspace of gptoss_attn_fwd: rotated k (fp16, [token][Hkv][64]), then at a
// 256-byte boundary each token's 32 (c cos, c sin) pairs ([token][32] float2).
static size_t fwd_ws_k_bytes(int32_t total_tokens, int32_t Hkv) {
  return (static_cast<size_t>(total_tokens) * Hkv * kHeadDim * 2 + 255) & ~static_cast<size_t>(255);
}

size_t gptoss_attn_fwd_workspace_size(int32_t total_tokens, int32_t Hkv, int32_t D) {
  if (total_tokens < 0 || Hkv <= 0 || D != kHeadDim) return 0;
  return fwd_ws_k_bytes(total_tokens, Hkv) + static_cast<size_t>(total_tokens) * kPairs * sizeof(float2);
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
  gptoss_status st = check_rope(rope, D);
  if (st != GPTOSS_OK) return st;
  const bool thd = cu_seqlens != nullptr;
  if (!thd && static_cast<int64_t>(B) * S != total_tokens) return GPTOSS_ERR_INVALID_ARG;
  if (total_tokens == 0 || B == 0 || S == 0) return GPTOSS_OK;
  if (!q || !k || !v || !sinks || !out) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(sq, !thd) || !strides_ok(sk, !thd) || !strides_ok(sv, !thd) || !strides_ok(so, !thd))
    return GPTOSS_ERR_INVALID_ARG;
  // with RoPE and a workspace, k is rotated once into it (fp16) instead of
  // once per work unit inside the kernel
  const bool k_pre = rope != nullptr && workspace != nullptr;
  if (k_pre && (workspace_bytes < gptoss_attn_fwd_workspace_size(total_tokens, Hkv, D) || !aligned16(workspace)))
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
  const uint64_t kb_stride = thd ? dimS * sk.tok * 2 : static_cast<uint64_t>(sk.batch) * 2;
  const uint64_t vb_stride = thd ? dimS * sv.tok * 2 : static_cast<uint64_t>(sv.batch) * 2;
  if (k_pre) {  // dense fp16 [B, S, Hkv, D] / [T, Hkv, D] in the workspace
    const uint64_t tok_b = static_cast<uint64_t>(Hkv) * kHeadDim * 2;
    st = make_tmap_4d(&p.tmap_k, workspace, kHeadDim, Hkv, dimS, dimB, kHeadDim * 2, tok_b,
                      thd ? dimS * tok_b : static_cast<uint64_t>(S) * tok_b, kHeadDim, 1, kFwdTile, 1, true);
  } else {
    st = make_tmap_4d(&p.tmap_k, k, kHeadDim, Hkv, dimS, dimB, sk.head * 2, sk.tok * 2,
                      kb_stride == 0 ? 16 : kb_stride, kHeadDim, 1, kFwdTile, 1);
  }
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_v, v, kHeadDim, Hkv, dimS, dimB, sv.head * 2, sv.tok * 2,
                         vb_stride == 0 ? 16 : vb_stride, kHeadDim, 1, kFwdTile, 1);
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
  if (rope != nullptr) yarn_table(*rope, &p.tab);
  else p.tab.enabled = 0;
  p.k_in_kernel = rope != nullptr && !k_pre;
  if (k_pre) {
    RopeQkParams rp;
    memset(&rp, 0, sizeof(rp));
    rp.k = static_cast<const __nv_bfloat16*>(k);
    rp.k_out = static_cast<__nv_bfloat16*>(workspace);  // fp16 bits (rope_qk_kernel<true>)
    rp.sk = sk;
    rp.sko.head = kHeadDim;
    rp.sko.tok = static_cast<int64_t>(Hkv) * kHeadDim;
    rp.sko.batch = thd ? 0 : static_cast<int64_t>(S) * Hkv * kHeadDim;
    rp.tm.positions = positions;
    rp.tm.cu_seqlens = cu_seqlens;
    rp.tm.nseq = B;
    rp.tm.S = thd ? 0 : S;
    rp.tm.ntok = total_tokens;
    rp.Hq = 0;
    rp.Hkv = Hkv;
    rp.tab = p.tab;
    rp.cs_out = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + fwd_ws_k_bytes(total_tokens, Hkv));
    p.cs_tab = rp.cs_out;
    const int rgrid = (total_tokens + kRopeTokensPerCta - 1) / kRopeTokensPerCta;
    rope_qk_kernel<true><<<rgrid, kRopeThreads, 0, as_stream(stream)>>>(rp);
    st = check_launch();
    if (st != GPTOSS_OK) return st;
  }
  const size_t smem = sizeof(FwdSmem) + 1024;
  if (cudaFuncSetAttribute(attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  attn_fwd_kernel<<<grid, kFwdThreads, smem, as_stream(stream)>>>(p);
  return check_launch();
}

size_t gptoss_attn_decode_workspace_size(int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D) {
  if (B <= 0 || Lmax <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D != kHeadDim) return 0;
  const int chunk = decode_chunk(B, Lmax, Hkv);
  const int64_t nsplit = (Lmax + chunk - 1) / chunk;
  const int64_t slots = static_cast<int64_t>(B) * Hkv * nsplit * (Hq / Hkv);
  return static_cast<size_t>(slots * (kHeadDim + 2) * sizeof(float));
}

}  // extern "C"

namespace {

// A paged cache: pools [num_blocks * block_size, Hkv, 64] and the block table.
struct PagedLayout {
  const int32_t* table;
  int32_t max_blocks, block_size, num_blocks;
};

// Decode over a contiguous cache [B, Lmax, Hkv, 64] (paged == nullptr) or a
// paged one (Lmax = max_blocks * block_size, the caches are the pools).
gptoss_status decode_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_seqlens,
                          const float* sinks, int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D,
                          int32_t window, float softmax_scale, const gptoss_rope_params* rope, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, struct CUstream_st* stream,
                          const PagedLayout* paged) {
  if (B < 0 || Lmax <= 0 || Hq <= 0 || Hkv <= 0 || window < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (Hq / Hkv > kDecMaxGroup) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  gptoss_status st = check_rope(rope, D);
  if (st != GPTOSS_OK) return st;
  if (B == 0) return GPTOSS_OK;
  if (!q || !k_cache || !v_cache || !cache_seqlens || !sinks || !out || !workspace) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace))
    return GPTOSS_ERR_INVALID_ARG;
  const size_t need = gptoss_attn_decode_workspace_size(B, Lmax, Hq, Hkv, D);
  if (need == 0 || workspace_bytes < need) return GPTOSS_ERR_INVALID_ARG;
  const int64_t rows = paged ? static_cast<int64_t>(paged->num_blocks) * paged->block_size
                             : static_cast<int64_t>(B) * Lmax;
  if (rows * Hkv * kHeadDim > (int64_t(1) << 40)) return GPTOSS_ERR_UNSUPPORTED;

  DecodeParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t tok_b = static_cast<uint64_t>(Hkv) * kHeadDim * 2;
  // contiguous: (d, head, slot, sequence); paged: (d, head, pool row, 1)
  const uint64_t d2 = paged ? static_cast<uint64_t>(rows) : static_cast<uint64_t>(Lmax);
  const uint64_t d3 = paged ? 1 : static_cast<uint64_t>(B);
  const uint64_t bat_b = paged ? tok_b * d2 : tok_b * Lmax;
  st = make_tmap_4d(&p.tmap_k, k_cache, kHeadDim, Hkv, d2, d3, kHeadDim * 2, tok_b, bat_b, kHeadDim, 1,
                    kDecTileKeys, 1);
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_v, v_cache, kHeadDim, Hkv, d2, d3, kHeadDim * 2, tok_b, bat_b, kHeadDim, 1,
                    kDecTileKeys, 1);
  if (st != GPTOSS_OK) return st;
  const int G = Hq / Hkv;
  const int chunk = decode_chunk(B, Lmax, Hkv);
  const int nsplit_max = (Lmax + chunk - 1) / chunk;
  const int span = window > 0 ? (window < Lmax ? window : Lmax) : Lmax;
  // a window that does not start on a 64-key boundary may touch one more tile,
  // still inside one split: chunks are multiples of 64 keys and at least 256
  const int nsplit = (span + chunk - 1) / chunk;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.seqlens = cache_seqlens;
  p.sinks = sinks;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = p.ws_o + static_cast<int64_t>(B) * Hkv * nsplit_max * G * kHeadDim;
  p.B = B;
  p.Lmax = Lmax;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.window = window;
  p.chunk = chunk;
  p.nsplit = nsplit_max;
  p.direct = nsplit == 1;  // e.g. window 128: one split per (sequence, kv head)
  if (paged) {
    p.block_table = paged->table;
    p.max_blocks = paged->max_blocks;
    p.block_size = paged->block_size;
    p.num_blocks = paged->num_blocks;
  }
  p.scale_log2 = softmax_scale * kLog2e;
  p.wait_ns = wait_limit_ns();
  if (rope != nullptr) yarn_table(*rope, &p.tab);
  else p.tab.enabled = 0;
  const size_t smem = sizeof(DecodeSmem) + 1024;
  if (cudaFuncSetAttribute(attn_decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return GPTOSS_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  attn_decode_split_kernel<<<dim3(Hkv, nsplit, B), kDecThreads, smem, s>>>(p);
  if (check_launch() != GPTOSS_OK) return GPTOSS_ERR_CUDA;
  if (p.direct) return GPTOSS_OK;
  attn_decode_merge_kernel<<<dim3(Hkv, B), 256, 0, s>>>(p);
  return check_launch();
}

gptoss_status check_paged(int32_t max_blocks, int32_t block_size, int32_t num_blocks) {
  if (max_blocks <= 0 || block_size <= 0 || num_blocks <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (block_size % kDecTileKeys) return GPTOSS_ERR_UNSUPPORTED;  // 64-key tiles must not straddle blocks
  if (static_cast<int64_t>(num_blocks) * block_size >= (int64_t(1) << 31) ||
      static_cast<int64_t>(max_blocks) * block_size >= (int64_t(1) << 31))
    return GPTOSS_ERR_UNSUPPORTED;
  return GPTOSS_OK;
}

}  // namespace

extern "C" {

gptoss_status gptoss_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* cache_seqlens, const float* sinks, int32_t B, int32_t Lmax,
                                 int32_t Hq, int32_t Hkv, int32_t D, int32_t window, float softmax_scale,
                                 const gptoss_rope_params* rope, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, struct CUstream_st* stream) {
  return decode_impl(q, k_cache, v_cache, cache_seqlens, sinks, B, Lmax, Hq, Hkv, D, window, softmax_scale, rope,
                     out, lse, workspace, workspace_bytes, stream, nullptr);
}

gptoss_status gptoss_attn_decode_paged(const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                       int32_t num_blocks, const int32_t* cache_seqlens, const float* sinks,
                                       int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t window,
                                       float softmax_scale, const gptoss_rope_params* rope, void* out, float* lse,
                                       void* workspace, size_t workspace_bytes, struct CUstream_st* stream) {
  gptoss_status st = check_paged(max_blocks, block_size, num_blocks);
  if (st != GPTOSS_OK) return st;
  if (B > 0 && block_table == nullptr) return GPTOSS_ERR_INVALID_ARG;
  const PagedLayout layout{block_table, max_blocks, block_size, num_blocks};
  return decode_impl(q, k_pool, v_pool, cache_seqlens, sinks, B, max_blocks * block_size, Hq, Hkv, D, window,
                     softmax_scale, rope, out, lse, workspace, workspace_bytes, stream, &layout);
}

gptoss_status gptoss_kv_append_paged(const void* k_new, const void* v_new, const int32_t* cache_seqlens,
                                     const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                     void* k_pool, void* v_pool, int32_t num_blocks, int32_t B, int32_t Hkv,
                                     int32_t D, const gptoss_rope_params* rope, struct CUstream_st* stream) {
  if (B < 0 || Hkv <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (Hkv * kPairs > 1024) return GPTOSS_ERR_UNSUPPORTED;
  gptoss_status st = check_paged(max_blocks, block_size, num_blocks);
  if (st != GPTOSS_OK) return st;
  st = check_rope(rope, D);
  if (st != GPTOSS_OK) return st;
  if (B == 0) return GPTOSS_OK;
  if (!k_new || !v_new || !cache_seqlens || !block_table || !k_pool || !v_pool) return GPTOSS_ERR_INVALID_ARG;
  AppendParams p;
  memset(&p, 0, sizeof(p));
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.seqlens = cache_seqlens;
  p.block_table = block_table;
  p.k_pool = static_cast<__nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<__nv_bfloat16*>(v_pool);
  p.B = B;
  p.Hkv = Hkv;
  p.max_blocks = max_blocks;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  if (rope != nullptr) yarn_table(*rope, &p.tab);
  else p.tab.enabled = 0;
  kv_append_paged_kernel<<<B, Hkv * kPairs, 0, as_stream(stream)>>>(p);
  return check_launch();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they decode:
// a serving loop that plans its memory once up front and may not call
// cudaMalloc (which can synchronise the device or fail under memory pressure),
// or a host runtime whose only device memory comes from its own fixed pools.
// For them the split-KV partials live in one file-scope device array of fixed
// size instead.  Every GPU that loads this library holds the array until the
// process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// The array's name is a host-side stand-in in host code: its device address
// comes from cudaGetSymbolAddress, once per device, with that device current.
void* g_scratch_addr[kNoAllocMaxDevices];
std::once_flag g_scratch_once[kNoAllocMaxDevices];
cudaError_t g_scratch_err[kNoAllocMaxDevices];

void* scratch_address(int device, gptoss_status* st) {
  if (device < 0 || device >= kNoAllocMaxDevices) {
    *st = GPTOSS_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::call_once(g_scratch_once[device], [device]() {
    void* ptr = nullptr;
    g_scratch_err[device] = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    g_scratch_addr[device] = ptr;
  });
  if (g_scratch_err[device] != cudaSuccess || g_scratch_addr[device] == nullptr) {
    *st = GPTOSS_ERR_CUDA;
    return nullptr;
  }
  *st = GPTOSS_OK;
  return g_scratch_addr[device];
}

}  // namespace

extern "C" gptoss_status gptoss_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                    const int32_t* cache_seqlens, const float* sinks, int32_t B,
                                                    int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D,
                                                    int32_t window, float softmax_scale,
                                                    const gptoss_rope_params* rope, void* out, float* lse,
                                                    struct CUstream_st* stream) {
  if (B == 0) return gptoss_attn_decode(q, k_cache, v_cache, cache_seqlens, sinks, B, Lmax, Hq, Hkv, D, window,
                                        softmax_scale, rope, out, lse, nullptr, 0, stream);
  const size_t need = gptoss_attn_decode_workspace_size(B, Lmax, Hq, Hkv, D);
  if (need == 0) return D != kHeadDim ? GPTOSS_ERR_UNSUPPORTED : GPTOSS_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return GPTOSS_ERR_UNSUPPORTED;  // partials exceed the fixed array
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return GPTOSS_ERR_CUDA;
  gptoss_status st = GPTOSS_OK;
  void* ws = scratch_address(device, &st);
  if (ws == nullptr) return st;
  return gptoss_attn_decode(q, k_cache, v_cache, cache_seqlens, sinks, B, Lmax, Hq, Hkv, D, window, softmax_scale,
                            rope, out, lse, ws, kNoAllocScratchBytes, stream);
}
