// host_util.cuh -- host-side helpers of libgptoss_attn: YaRN tables, argument
// checks, TMA tensor-map encoding.  No allocation, no synchronisation.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "gptoss.h"

namespace gptoss {

constexpr int kHeadDim = 64;
constexpr int kPairs = kHeadDim / 2;
// the larger head size some entry points also take (RoPE, prefill, decode)
constexpr int kMaxHeadDim = 128;
constexpr int kMaxPairs = kMaxHeadDim / 2;
constexpr float kLog2e = 1.4426950408889634f;  // log2(e)
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)

// Per-launch rotary table: inverse frequencies in double plus the
// concentration.  Passed to kernels by value (524 bytes).
struct RopeTable {
  double inv_freq[kMaxPairs];
  float conc;
  int enabled;  // 0: inputs already rotated, nothing to do
  int R;        // rotary pairs, rotary_dim / 2: features [0, 2R) rotate in pairs (j, j + R), the rest pass through
};

// YaRN inverse frequencies and concentration (RotaryEmbedding on the NeMo
// AutoModel gpt_oss.rope_utils page, _compute_concentration_and_inv_freq,
// after the YaRN paper arXiv 2309.00071):
//   f_j = base^(-2j/rdim);  factor <= 1: inv_freq = f, c = 1;
//   else c = 0.1 ln(factor) + 1; d(turns) = (rdim/2) ln(L0 / (2 pi turns)) / ln(base);
//   ramp_j = clamp((j - d(beta)) / (d(alpha) - d(beta)), 0, 1);
//   inv_freq_j = f_j (1 - ramp_j) + (f_j / factor) ramp_j.
inline void yarn_table(const gptoss_rope_params& rp, RopeTable* t) {
  const int rdim = rp.rotary_dim;
  const int half = rdim / 2;
  const double two_pi = 6.283185307179586476925286766559;
  for (int j = 0; j < kMaxPairs; ++j) t->inv_freq[j] = 0.0;
  t->R = half;
  const double lnb = log(rp.base);
  if (rp.factor <= 1.0) {
    for (int j = 0; j < half; ++j) t->inv_freq[j] = exp(-2.0 * j / rdim * lnb);
    t->conc = 1.0f;
  } else {
    const double d_lo = 0.5 * rdim * log(rp.initial_context / (rp.ntk_beta * two_pi)) / lnb;
    const double d_hi = 0.5 * rdim * log(rp.initial_context / (rp.ntk_alpha * two_pi)) / lnb;
    for (int j = 0; j < half; ++j) {
      const double f = exp(-2.0 * j / rdim * lnb);
      double r = (j - d_lo) / (d_hi - d_lo);
      r = r < 0.0 ? 0.0 : (r > 1.0 ? 1.0 : r);
      t->inv_freq[j] = f * (1.0 - r) + (f / rp.factor) * r;
    }
    t->conc = static_cast<float>(0.1 * log(rp.factor) + 1.0);
  }
  t->enabled = 1;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(struct CUstream_st* s) { return reinterpret_cast<cudaStream_t>(s); }

inline gptoss_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? GPTOSS_OK : GPTOSS_ERR_CUDA;
}

// Validates rope params.  rotary_dim must be even and at most head_dim;
// kernels that take partial rotary (allow_partial) need it a multiple of 16
// (whole 16-byte chunks of pairs), the others need rotary_dim == head_dim.
inline gptoss_status check_rope(const gptoss_rope_params* rp, int D, bool allow_partial = false) {
  if (rp == nullptr) return GPTOSS_OK;
  if (!(rp->base > 1.0) || !(rp->factor > 0.0) || rp->initial_context <= 0) return GPTOSS_ERR_INVALID_ARG;
  if (rp->factor > 1.0 && !(rp->ntk_alpha > 0.0 && rp->ntk_beta > rp->ntk_alpha)) return GPTOSS_ERR_INVALID_ARG;
  if (rp->rotary_dim <= 0 || (rp->rotary_dim & 1) || rp->rotary_dim > D) return GPTOSS_ERR_INVALID_ARG;
  if (rp->rotary_dim != D && (!allow_partial || (rp->rotary_dim % 16) != 0)) return GPTOSS_ERR_UNSUPPORTED;
  return GPTOSS_OK;
}

// Strides: positive multiples of 8 elements (16 bytes), batch ignored for THD.
inline bool strides_ok(const gptoss_strides& s, bool bshd) {
  if (s.tok <= 0 || s.head <= 0 || (s.tok & 7) || (s.head & 7)) return false;
  if (bshd && (s.batch < 0 || (s.batch & 7))) return false;
  return true;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library links no driver stub).
// ---------------------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 4-D bf16 (or fp16) map (dims innermost first: d, head, token, batch) with a 128-byte
// swizzle; out-of-range rows read as zeros.
inline gptoss_status make_tmap_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                                       uint64_t d2, uint64_t d3, uint64_t s1_bytes, uint64_t s2_bytes,
                                       uint64_t s3_bytes, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3,
                                       bool fp16 = false) {
  auto fn = encode_fn();
  if (fn == nullptr) return GPTOSS_ERR_CUDA;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {s1_bytes, s2_bytes, s3_bytes};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTOSS_OK : GPTOSS_ERR_INVALID_ARG;
}

// Default wait limit of the device-side pipeline waits, in nanoseconds.
inline uint64_t& wait_limit_ns() {
  static uint64_t v = 2000000000ull;  // 2 s
  return v;
}

}  // namespace gptoss
