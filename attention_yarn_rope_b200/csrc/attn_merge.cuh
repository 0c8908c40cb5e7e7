// attn_merge.cuh -- log-sum-exp merge of key-block results (gptoss_attn_merge),
// the last step of context parallelism for the full-context layers.
//
// Rule: the sink attention of the gpt_oss.layers page (the sink adds to the
// softmax denominator only) over keys split into disjoint blocks b.  With
// lse_b = log sum_{j in b} exp(s_j) and o_b the block's own normalised
// output (gptoss_attn_fwd_block, no sink),
//     Z = exp(sink) + sum_b exp(lse_b),   o = sum_b exp(lse_b) o_b / Z,
// so the sink enters once, here.  Context parallelism itself is the cp_size /
// cp_rank arguments of apply_rotary_emb_qk on the gpt_oss.rope_utils page.
//
// Design (HBM-bound elementwise op): 16 threads per (batch row, token, head)
// row, each reading 4 of the row's 64 features from every block with one
// float4 load (the blocks' rows are contiguous 256-byte lines) and writing 4
// bf16 values of the output.
#pragma once

#include "host_util.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

struct MergeParams {
  const float* outs;   // [n][B][S][Hq][64] fp32
  const float* lses;   // [n][B][Hq][S] fp32 (natural log)
  const float* sinks;  // [Hq] fp32, nullable (no sink)
  __nv_bfloat16* out;  // bf16 [B][S][Hq][64] with strides so
  gptoss_strides so;
  float* lse;          // nullable: [B][Hq][S]
  int n, B, S, Hq;
};

constexpr int kMergeThreads = 256;
constexpr int kMergeRowsPerCta = kMergeThreads / 16;

__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(const __grid_constant__ MergeParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.S * p.Hq;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeRowsPerCta + threadIdx.x / 16;
  if (row >= rows) return;
  const int l16 = threadIdx.x & 15;
  const int h = static_cast<int>(row % p.Hq);
  const int64_t bs = row / p.Hq;  // b * S + s
  const int s = static_cast<int>(bs % p.S);
  const int b = static_cast<int>(bs / p.S);
  const int64_t lse_idx = (static_cast<int64_t>(b) * p.Hq + h) * p.S + s;
  const int64_t blk_lse = static_cast<int64_t>(p.B) * p.Hq * p.S;
  const int64_t blk_out = rows * kHeadDim;
  const float sink = p.sinks != nullptr ? __ldg(p.sinks + h) : -INFINITY;
  float m = sink;
  for (int i = 0; i < p.n; ++i) m = fmaxf(m, __ldg(p.lses + i * blk_lse + lse_idx));
  float z = sink == -INFINITY ? 0.f : expf(sink - m);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < p.n; ++i) {
    const float l = __ldg(p.lses + i * blk_lse + lse_idx);
    if (l == -INFINITY) continue;  // a block this row sees no key of
    const float w = expf(l - m);
    z += w;
    const float4 o = __ldg(reinterpret_cast<const float4*>(p.outs + i * blk_out + row * kHeadDim) + l16);
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  const float inv = 1.f / z;
  uint2 v;
  v.x = pack_bf16(acc.x * inv, acc.y * inv);
  v.y = pack_bf16(acc.z * inv, acc.w * inv);
  __nv_bfloat16* dst = p.out + static_cast<int64_t>(b) * p.so.batch + static_cast<int64_t>(s) * p.so.tok +
                       static_cast<int64_t>(h) * p.so.head + 4 * l16;
  *reinterpret_cast<uint2*>(dst) = v;
  if (p.lse != nullptr && l16 == 0) p.lse[lse_idx] = m + logf(z);
}

}  // namespace gptoss

extern "C" gptoss_status gptoss_attn_merge(const float* outs, const float* lses, int32_t n_blocks,
                                           const float* sinks, int32_t B, int32_t S, int32_t Hq, int32_t D,
                                           void* out, gptoss_strides so, float* lse, struct CUstream_st* stream) {
  using namespace gptoss;
  if (n_blocks < 0 || B < 0 || S < 0 || Hq <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (D != kHeadDim) return GPTOSS_ERR_UNSUPPORTED;
  if (n_blocks == 0 || B == 0 || S == 0) return n_blocks == 0 && B > 0 && S > 0 ? GPTOSS_ERR_INVALID_ARG : GPTOSS_OK;
  if (!outs || !lses || !out) return GPTOSS_ERR_INVALID_ARG;
  // 8-byte output stores: bf16 rows start on 8-byte boundaries
  if ((reinterpret_cast<uintptr_t>(out) & 7u) || (reinterpret_cast<uintptr_t>(outs) & 15u))
    return GPTOSS_ERR_INVALID_ARG;
  if (!strides_ok(so, true)) return GPTOSS_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * S * Hq;
  const int64_t grid = (rows + kMergeRowsPerCta - 1) / kMergeRowsPerCta;
  if (grid > INT32_MAX) return GPTOSS_ERR_UNSUPPORTED;
  MergeParams p;
  p.outs = outs;
  p.lses = lses;
  p.sinks = sinks;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.so = so;
  p.lse = lse;
  p.n = n_blocks;
  p.B = B;
  p.S = S;
  p.Hq = Hq;
  attn_merge_kernel<<<static_cast<unsigned>(grid), kMergeThreads, 0, as_stream(stream)>>>(p);
  return check_launch();
}
