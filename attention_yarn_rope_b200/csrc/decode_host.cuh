// decode_host.cuh -- host side of the decode entry points of libgptoss_attn
// (declared in include/gptoss.h): split-KV decode over a contiguous or paged
// cache, appending new tokens to a paged cache, and decode without a
// caller-provided workspace.  Included once, at the end of gptoss_lib.cu (the
// library is one translation unit, so the device status word is shared).
#pragma once

#include <cuda_runtime.h>

#include <mutex>

#include "attn_decode.cuh"
#include "gptoss.h"
#include "host_util.cuh"

using namespace gptoss;

extern "C" {

size_t gptoss_attn_decode_workspace_size(int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D) {
  if (B <= 0 || Lmax <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || (D != kHeadDim && D != kMaxHeadDim)) return 0;
  const int chunk = decode_chunk(B, Lmax, Hkv);
  const int64_t nsplit = (Lmax + chunk - 1) / chunk;
  const int64_t slots = static_cast<int64_t>(B) * Hkv * nsplit * (Hq / Hkv);
  return static_cast<size_t>(slots * (D + 2) * sizeof(float));
}

}  // extern "C"

namespace {

// A paged cache: pools [num_blocks * block_size, Hkv, D] and the block table.
struct PagedLayout {
  const int32_t* table;
  int32_t max_blocks, block_size, num_blocks;
};

// Decode over a contiguous cache [B, Lmax, Hkv, D] (paged == nullptr) or a
// paged one (Lmax = max_blocks * block_size, the caches are the pools).
gptoss_status decode_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* cache_seqlens,
                          const float* sinks, int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv, int32_t D,
                          int32_t window, float softmax_scale, const gptoss_rope_params* rope, void* out,
                          float* lse, void* workspace, size_t workspace_bytes, struct CUstream_st* stream,
                          const PagedLayout* paged, int32_t q_len) {
  if (q_len <= 0) return GPTOSS_ERR_INVALID_ARG;
  // B x q_len virtual sequences (query token i of cache row b)
  const int64_t BQ = static_cast<int64_t>(B) * q_len;
  if (BQ > 65535) return GPTOSS_ERR_UNSUPPORTED;  // grid z / y limit
  if (B < 0 || Lmax <= 0 || Hq <= 0 || Hkv <= 0 || window < 0) return GPTOSS_ERR_INVALID_ARG;
  if (Hq % Hkv) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim && D != kMaxHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (Hq / Hkv > kDecMaxGroup) return GPTOSS_ERR_UNSUPPORTED;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return GPTOSS_ERR_INVALID_ARG;
  gptoss_status st = check_rope(rope, D, /*allow_partial=*/true);
  if (st != GPTOSS_OK) return st;
  if (B == 0) return GPTOSS_OK;
  if (!q || !k_cache || !v_cache || !cache_seqlens || !sinks || !out || !workspace) return GPTOSS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace))
    return GPTOSS_ERR_INVALID_ARG;
  const size_t need = gptoss_attn_decode_workspace_size(static_cast<int32_t>(BQ), Lmax, Hq, Hkv, D);
  if (need == 0 || workspace_bytes < need) return GPTOSS_ERR_INVALID_ARG;
  const int64_t rows = paged ? static_cast<int64_t>(paged->num_blocks) * paged->block_size
                             : static_cast<int64_t>(B) * Lmax;
  if (rows * Hkv * D > (int64_t(1) << 40)) return GPTOSS_ERR_UNSUPPORTED;

  DecodeParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t tok_b = static_cast<uint64_t>(Hkv) * D * 2;
  // contiguous: (d, head, slot, sequence); paged: (d, head, pool row, 1)
  const uint64_t d2 = paged ? static_cast<uint64_t>(rows) : static_cast<uint64_t>(Lmax);
  const uint64_t d3 = paged ? 1 : static_cast<uint64_t>(B);
  const uint64_t bat_b = paged ? tok_b * d2 : tok_b * Lmax;
  // boxes of 64 features (a D = 128 row is two)
  st = make_tmap_4d(&p.tmap_k, k_cache, D, Hkv, d2, d3, D * 2, tok_b, bat_b, kHeadDim, 1, kDecTileKeys, 1);
  if (st != GPTOSS_OK) return st;
  st = make_tmap_4d(&p.tmap_v, v_cache, D, Hkv, d2, d3, D * 2, tok_b, bat_b, kHeadDim, 1, kDecTileKeys, 1);
  if (st != GPTOSS_OK) return st;
  const int G = Hq / Hkv;
  // tokens per CTA: as many as fill one 16-row M fragment, or two when q_len
  // needs more than one fragment's worth
  const int rm = q_len > 16 / G ? 2 : 1;
  const int tpc = q_len < 16 * rm / G ? q_len : 16 * rm / G;
  const int n_slices = (q_len + tpc - 1) / tpc;
  const int chunk = decode_chunk(static_cast<int>(BQ), Lmax, Hkv);
  const int nsplit_max = (Lmax + chunk - 1) / chunk;
  // a CTA's tokens see the union of their key ranges: window + tpc - 1 keys
  const int64_t span_w = static_cast<int64_t>(window) + tpc - 1;
  const int span = window > 0 ? (span_w < Lmax ? static_cast<int>(span_w) : Lmax) : Lmax;
  // a window that does not start on a 64-key boundary may touch one more tile,
  // still inside one split: chunks are multiples of 64 keys and at least 256
  const int nsplit = (span + chunk - 1) / chunk;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.seqlens = cache_seqlens;
  p.sinks = sinks;
  p.ws_o = static_cast<float*>(workspace);
  p.ws_ml = p.ws_o + BQ * Hkv * nsplit_max * G * D;
  p.B = B;
  p.q_len = q_len;
  p.tpc = tpc;
  p.n_slices = n_slices;
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
  const bool d128 = D == kMaxHeadDim;
  // one split of at most four 64-key tiles (a 128-key window) takes the short
  // K / V ring: a smaller CTA, more of them resident on an SM, and the range
  // needs no deeper prefetch
  const bool short_ring = p.direct && span <= 4 * kDecTileKeys;
  size_t smem;
  void (*kernel)(DecodeParams);
  if (d128) {
    smem = short_ring ? sizeof(DecodeSmem<kMaxHeadDim, kDecShortStages>) : sizeof(DecodeSmem<kMaxHeadDim>);
    kernel = short_ring ? (rm == 1 ? attn_decode_split_kernel<1, kMaxHeadDim, kDecShortStages>
                                   : attn_decode_split_kernel<2, kMaxHeadDim, kDecShortStages>)
                        : (rm == 1 ? attn_decode_split_kernel<1, kMaxHeadDim> : attn_decode_split_kernel<2, kMaxHeadDim>);
  } else {
    smem = short_ring ? sizeof(DecodeSmem<kHeadDim, kDecShortStages>) : sizeof(DecodeSmem<kHeadDim>);
    kernel = short_ring ? (rm == 1 ? attn_decode_split_kernel<1, kHeadDim, kDecShortStages>
                                   : attn_decode_split_kernel<2, kHeadDim, kDecShortStages>)
                        : (rm == 1 ? attn_decode_split_kernel<1, kHeadDim> : attn_decode_split_kernel<2, kHeadDim>);
  }
  smem += 1024;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return GPTOSS_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const dim3 grid(Hkv, nsplit, static_cast<unsigned>(static_cast<int64_t>(B) * n_slices));
  kernel<<<grid, kDecThreads, smem, s>>>(p);
  if (check_launch() != GPTOSS_OK) return GPTOSS_ERR_CUDA;
  if (p.direct) return GPTOSS_OK;
  if (d128) attn_decode_merge_kernel<kMaxHeadDim><<<dim3(Hkv, static_cast<unsigned>(BQ)), 256, 0, s>>>(p);
  else attn_decode_merge_kernel<kHeadDim><<<dim3(Hkv, static_cast<unsigned>(BQ)), 256, 0, s>>>(p);
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
                     out, lse, workspace, workspace_bytes, stream, nullptr, 1);
}

gptoss_status gptoss_attn_decode_paged(const void* q, const void* k_pool, const void* v_pool,
                                       const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                       int32_t num_blocks, const int32_t* cache_seqlens, const float* sinks,
                                       int32_t B, int32_t q_len, int32_t Hq, int32_t Hkv, int32_t D,
                                       int32_t window, float softmax_scale, const gptoss_rope_params* rope,
                                       void* out, float* lse, void* workspace, size_t workspace_bytes,
                                       struct CUstream_st* stream) {
  gptoss_status st = check_paged(max_blocks, block_size, num_blocks);
  if (st != GPTOSS_OK) return st;
  if (B > 0 && block_table == nullptr) return GPTOSS_ERR_INVALID_ARG;
  const PagedLayout layout{block_table, max_blocks, block_size, num_blocks};
  return decode_impl(q, k_pool, v_pool, cache_seqlens, sinks, B, max_blocks * block_size, Hq, Hkv, D, window,
                     softmax_scale, rope, out, lse, workspace, workspace_bytes, stream, &layout, q_len);
}

gptoss_status gptoss_kv_append_paged(const void* k_new, const void* v_new, const int32_t* cache_seqlens,
                                     const int32_t* block_table, int32_t max_blocks, int32_t block_size,
                                     void* k_pool, void* v_pool, int32_t num_blocks, int32_t B, int32_t q_len,
                                     int32_t Hkv, int32_t D, const gptoss_rope_params* rope,
                                     struct CUstream_st* stream) {
  if (B < 0 || q_len <= 0 || Hkv <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (q_len > 65535) return GPTOSS_ERR_UNSUPPORTED;
  if (D != kHeadDim && D != kMaxHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (Hkv * (D / 2) > 1024) return GPTOSS_ERR_UNSUPPORTED;
  gptoss_status st = check_paged(max_blocks, block_size, num_blocks);
  if (st != GPTOSS_OK) return st;
  st = check_rope(rope, D, /*allow_partial=*/true);
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
  p.q_len = q_len;
  p.Hkv = Hkv;
  p.D = D;
  p.max_blocks = max_blocks;
  p.block_size = block_size;
  p.num_blocks = num_blocks;
  if (rope != nullptr) yarn_table(*rope, &p.tab);
  else p.tab.enabled = 0;
  kv_append_paged_kernel<<<dim3(B, q_len), Hkv * (D / 2), 0, as_stream(stream)>>>(p);
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
constexpr int kScratchCacheSlots = 16;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// In host code the array's name is a host-side stand-in, not a device
// address.  The device address belongs to the CUDA context the library's
// module is loaded into -- not to a device number: after cudaDeviceReset, or
// with a non-primary driver context current, an address remembered per device
// would be stale.  So the address is looked up with cudaGetSymbolAddress
// (which allocates nothing) on the first call in each context, with that
// context current, and remembered under the context's unique id (cuCtxGetId;
// a process never reuses an id).  A full cache forgets its oldest entry; a
// forgotten context just looks its address up again.
struct ScratchSlot {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch_slots[kScratchCacheSlots];
int g_scratch_used = 0, g_scratch_next = 0;

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

void* scratch_address(gptoss_status* st) {
  static const PFN_cuCtxGetCurrent_v4000 get_current = driver_fn<PFN_cuCtxGetCurrent_v4000>("cuCtxGetCurrent");
  static const PFN_cuCtxGetId_v12000 get_id = driver_fn<PFN_cuCtxGetId_v12000>("cuCtxGetId");
  *st = GPTOSS_ERR_CUDA;
  if (get_current == nullptr || get_id == nullptr) return nullptr;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return nullptr;
  void* addr = nullptr;
  if (ctx == nullptr) {
    // no context current yet: the runtime binds the current device's primary
    // context while it resolves the symbol
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess) return nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  for (int i = 0; i < g_scratch_used; ++i)
    if (g_scratch_slots[i].ctx_id == id) {
      *st = GPTOSS_OK;
      return g_scratch_slots[i].addr;
    }
  if (addr == nullptr && cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess) return nullptr;
  if (addr == nullptr) return nullptr;
  const int slot = g_scratch_used < kScratchCacheSlots ? g_scratch_used++ : g_scratch_next++ % kScratchCacheSlots;
  g_scratch_slots[slot] = ScratchSlot{id, addr};
  *st = GPTOSS_OK;
  return addr;
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
  if (need == 0) return D != kHeadDim && D != kMaxHeadDim ? GPTOSS_ERR_UNSUPPORTED : GPTOSS_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return GPTOSS_ERR_UNSUPPORTED;  // partials exceed the fixed array
  gptoss_status st = GPTOSS_OK;
  void* ws = scratch_address(&st);
  if (ws == nullptr) return st;
  return gptoss_attn_decode(q, k_cache, v_cache, cache_seqlens, sinks, B, Lmax, Hq, Hkv, D, window, softmax_scale,
                            rope, out, lse, ws, kNoAllocScratchBytes, stream);
}
