// fwd128.cuh -- the prefill kernel for head size 128 (gptoss_attn_fwd, D = 128).
//
// Same method and pipeline as the D = 64 kernel (fwd_pipeline.cuh: sink
// attention of the gpt_oss.layers page, RoPE of the gpt_oss.rope_utils page
// fused into the Q tile load), one head per work unit.  A head's S (128
// columns), fp16 P (64) and O (128) take 320 of the 512 tensor-memory
// columns, so two heads no longer fit beside each other; with twice the
// tensor-core work per score, one softmax warpgroup per CTA keeps the tensor
// core and the MUFU unit about equally busy.
//
// Tiles: every 128-row tile of q, k or v is two 16 KB halves (features
// [0, 64) and [64, 128)), each a 128B-swizzled 128 x 64 box of the same
// tensor maps as the D = 64 kernel.
//   S  = Q K^T   (SS, M128 N128, 2 halves x 4 x K16, one accumulator)
//   O += P V     (TS, M128 N128, 8 x K16: the two feature halves of V are
//                 consecutive 128B-swizzle atoms along N, 16 KB apart;
//                 measured 1.2 % faster on full causal and 4.4 % on the
//                 128-key window than two N64 products per K step)
// Tensor memory: three S buffers [0, 384) (P over the first half of its S,
// product t in buffer t mod 3), O [384, 512).
// Warps: 0-3 rope (Q rotated in place: pair (j, j + 64) is word m of the
// two halves at the same swizzled position), 4-7 softmax (fwd_softmax.cuh,
// head slot 0), 8 K / V producer, 9 QK^T issuer and tensor-memory owner,
// 10 P V issuer, 11 Q producer.
#pragma once

#include "fwd_common.cuh"
#include "fwd_softmax.cuh"

namespace gptoss {

constexpr int kF128Threads = 384;
constexpr int kF128LaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr int kF128Stages = 2;        // K / V ring
constexpr int kF128QStages = 2;       // Q ring
constexpr uint32_t kF128RegsSoftmax = 232, kF128RegsRope = 80, kF128RegsOther = 56;
static_assert(128 * (kF128RegsSoftmax + kF128RegsRope + kF128RegsOther) <= kF128Threads * kF128LaunchRegs,
              "register split must fit in the launch allocation");

struct __align__(1024) Fwd128Smem {
  uint8_t q[kF128QStages][2][kFwdTileBytes];  // [stage][feature half], rotated in place to fp16
  uint8_t k[kF128Stages][2][kFwdTileBytes];   // fp16 (workspace)
  uint8_t v[kF128Stages][2][kFwdTileBytes];
  uint64_t q_loaded[kF128QStages], q_full[kF128QStages], q_empty[kF128QStages];
  uint64_t k_full[kF128Stages], k_empty[kF128Stages];
  uint64_t v_full[kF128Stages], v_empty[kF128Stages];
  uint64_t s_full[2][kSBufs], p_full[kSBufs], s_empty[kSBufs];  // as in FwdSmem (slot 0 of s_full only)
  uint64_t o_done[2];                                         // slot 0 only (the softmax role indexes a slot)
  uint64_t s_free[2];                                         // unused (three-buffer layout)
  uint64_t mma_final[2];
  uint32_t tmem_base;
};

__device__ __forceinline__ void fwd128_producer_kv_role(const FwdParams& p, Fwd128Smem& sm) {
  tma_prefetch_desc(&p.tmap_k);
  tma_prefetch_desc(&p.tmap_v);
  const bool thd = p.cu_seqlens != nullptr;
  uint32_t kv_it = 0, k_issued = 0, v_issued = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit<false>(p, u, wu)) continue;
    const int tok0 = thd ? wu.seq_start : 0;
    const int bc = thd ? 0 : wu.b;
    for (int j = 0; j < wu.n_kt; ++j, ++kv_it) {
      const int s = kv_it % kF128Stages;
      const uint32_t ph = ((kv_it / kF128Stages) & 1) ^ 1;
      const int key_row = tok0 + (wu.j_lo + j) * kFwdTile;
      if (!mbar_wait(&sm.k_empty[s], ph, p.wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.k_full[s], 2 * kFwdTileBytes);
      tma_load_4d(sm.k[s][0], &p.tmap_k, &sm.k_full[s], 0, wu.g, key_row, bc);
      tma_load_4d(sm.k[s][1], &p.tmap_k, &sm.k_full[s], 64, wu.g, key_row, bc);
      k_issued = kv_it + 1;
      if (!mbar_wait(&sm.v_empty[s], ph, p.wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.v_full[s], 2 * kFwdTileBytes);
      tma_load_4d(sm.v[s][0], &p.tmap_v, &sm.v_full[s], 0, wu.g, key_row, bc);
      tma_load_4d(sm.v[s][1], &p.tmap_v, &sm.v_full[s], 64, wu.g, key_row, bc);
      v_issued = kv_it + 1;
    }
  }
  // the copies of the last stages must land before the CTA exits
  for (uint32_t it = k_issued > kF128Stages ? k_issued - kF128Stages : 0; it < k_issued; ++it)
    mbar_wait(&sm.k_full[it % kF128Stages], (it / kF128Stages) & 1, p.wait_ns);
  for (uint32_t it = v_issued > kF128Stages ? v_issued - kF128Stages : 0; it < v_issued; ++it)
    mbar_wait(&sm.v_full[it % kF128Stages], (it / kF128Stages) & 1, p.wait_ns);
}

__device__ __forceinline__ void fwd128_producer_q_role(const FwdParams& p, Fwd128Smem& sm) {
  tma_prefetch_desc(&p.tmap_q);
  const bool thd = p.cu_seqlens != nullptr;
  uint32_t i = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit<false>(p, u, wu)) continue;
    const int qs = i % kF128QStages;
    if (!mbar_wait(&sm.q_empty[qs], ((i / kF128QStages) & 1) ^ 1, p.wait_ns)) break;
    mbar_arrive_expect_tx(&sm.q_loaded[qs], 2 * kFwdTileBytes);
    const int tok = (thd ? wu.seq_start : 0) + wu.q0;
    const int bc = thd ? 0 : wu.b;
    tma_load_4d(sm.q[qs][0], &p.tmap_q, &sm.q_loaded[qs], 0, wu.h0, tok, bc);
    tma_load_4d(sm.q[qs][1], &p.tmap_q, &sm.q_loaded[qs], 64, wu.h0, tok, bc);
    ++i;
  }
  for (uint32_t it = i > kF128QStages ? i - kF128QStages : 0; it < i; ++it)
    mbar_wait(&sm.q_loaded[it % kF128QStages], (it / kF128QStages) & 1, p.wait_ns);
}

// Rotates (or, with the identity table, converts) the Q tile of a unit in
// place.  Thread (w, l) owns words m = l % 16 and m + 16 (features 2m, 2m+1)
// of both halves in rows ro, ro + 8, .., ro + 120 (ro = w + 4 (l / 16)):
// word m of half 0 holds pairs 2m, 2m+1 and word m of half 1 their partners
// 2m + 64, 2m + 65.  Angles: the row-ro seeds from the per-token table
// times (cos 8f, sin 8f)^k, or every row's own table entries with explicit
// positions.  Rows at or past n_valid are only converted.
__device__ __forceinline__ void fwd128_rope_role(const FwdParams& p, Fwd128Smem& sm) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int m0 = l & 15;
  const int ro = w + 4 * (l >> 4);
  const bool explicit_pos = p.positions != nullptr;
  const bool thd = p.cu_seqlens != nullptr;
  float2 step[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) step[a] = rope_cs(8, p.tab.inv_freq[2 * (m0 + 16 * (a >> 1)) + (a & 1)], 1.f);
  const float2 one = make_float2(1.f, 0.f);
  uint32_t i = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit<false>(p, u, wu)) continue;
    const int qb = i % kF128QStages;
    if (!mbar_wait_warp_relaxed(&sm.q_loaded[qb], (i / kF128QStages) & 1, p.wait_ns)) return;
    const int n_valid = min(kFwdTile, wu.L - wu.q0);
    const int64_t tok_q0 = (thd ? wu.seq_start : static_cast<int64_t>(wu.b) * p.S) + wu.q0;
    const float4* row_cs = reinterpret_cast<const float4*>(p.cs_tab + tok_q0 * (2 * kPairs));  // 64 pairs per token
    float2 c[4] = {one, one, one, one};
    if (!explicit_pos && ro < n_valid) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 v = __ldg(row_cs + 32 * ro + m0 + 16 * h);
        c[2 * h] = make_float2(v.x, v.y);
        c[2 * h + 1] = make_float2(v.z, v.w);
      }
    }
    uint8_t* t0 = sm.q[qb][0];
    uint8_t* t1 = sm.q[qb][1];
#pragma unroll 1
    for (int kk = 0; kk < 16; ++kk) {
      const int r = ro + 8 * kk;
      float2 a[4] = {one, one, one, one};
      if (r < n_valid) {
        if (explicit_pos) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 v = __ldg(row_cs + 32 * r + m0 + 16 * h);
            a[2 * h] = make_float2(v.x, v.y);
            a[2 * h + 1] = make_float2(v.z, v.w);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) a[e] = c[e];
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t off = sw128_word(r, 2 * (m0 + 16 * h));
        uint32_t* lo = reinterpret_cast<uint32_t*>(t0 + off);
        uint32_t* hi = reinterpret_cast<uint32_t*>(t1 + off);
        uint32_t x = *lo, y = *hi;
        rotate_words(x, y, a[2 * h], a[2 * h + 1]);
        *lo = x;
        *hi = y;
      }
      if (!explicit_pos) {
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] = cmul(c[e], step[e]);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(&sm.q_full[qb]);
    ++i;
  }
}

// S = Q K^T: both feature halves accumulate into the one 128-column S.
__device__ __forceinline__ void fwd128_mma_s_role(const FwdParams& p, Fwd128Smem& sm, uint32_t tmem) {
  constexpr uint32_t idesc_s = idesc_f16_f32(128, 128);
  uint32_t t = 0, kv_it = 0, i = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit<false>(p, u, wu)) continue;
    const int qb = i % kF128QStages;
    if (!mbar_wait(&sm.q_full[qb], (i / kF128QStages) & 1, p.wait_ns)) break;
    for (int j = 0; j < wu.n_kt; ++j, ++t, ++kv_it) {
      const int s = kv_it % kF128Stages;
      if (!mbar_wait(&sm.k_full[s], (kv_it / kF128Stages) & 1, p.wait_ns)) { ok = false; break; }
      // product t into S buffer t mod 3, once product t - 3's P V has read its P
      const uint32_t b = t % kSBufs;
      if (t >= kSBufs && !mbar_wait(&sm.s_empty[b], ((t / kSBufs) - 1) & 1, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint64_t qdesc = sw128_desc(smem_u32(sm.q[qb][hf]));
        const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s][hf]));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + b * 128, qdesc + static_cast<uint64_t>(kk * 2), kdesc + static_cast<uint64_t>(kk * 2),
                 idesc_s, (hf | kk) > 0 ? 1u : 0u);
      }
      mma_commit(&sm.s_full[0][b]);
      mma_commit(&sm.k_empty[s]);
      if (j == wu.n_kt - 1) mma_commit(&sm.q_empty[qb]);
    }
    ++i;
  }
  mma_commit(&sm.mma_final[0]);
  mbar_wait(&sm.mma_final[0], 0, p.wait_ns);
}

// O += P V (TS: P from tensor memory, V read N-major, both feature halves in
// one N = 128 product); the first tile of a unit starts O from zero.
__device__ __forceinline__ void fwd128_mma_pv_role(const FwdParams& p, Fwd128Smem& sm, uint32_t tmem) {
  constexpr uint32_t idesc_o = idesc_f16_f32(128, 128, true);
  constexpr uint32_t colO = kColO;  // O: columns 384 .. 511
  uint32_t t = 0, kv_it = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit<false>(p, u, wu)) continue;
    for (int j = 0; j < wu.n_kt; ++j, ++t, ++kv_it) {
      const int s = kv_it % kF128Stages;
      if (!mbar_wait(&sm.v_full[s], (kv_it / kF128Stages) & 1, p.wait_ns)) { ok = false; break; }
      const uint32_t b = t % kSBufs, colP = b * 128;  // P sits over the S it came from
      if (!mbar_wait(&sm.p_full[b], (t / kSBufs) & 1, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      // one N = 128 product per K step: the second 64-feature half of V is
      // the next 128B-swizzle atom along N, 16 KB on (leading byte offset)
      const uint64_t vdesc = (sw128_desc(smem_u32(sm.v[s][0])) & ~(static_cast<uint64_t>(0x3FFF) << 16)) |
                             (static_cast<uint64_t>(kFwdTileBytes >> 4) << 16);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + colO, tmem + colP + kk * 8, vdesc + static_cast<uint64_t>(kk * 128), idesc_o,
               (j == 0 && kk == 0) ? 0u : 1u);
      mma_commit(&sm.o_done[0]);
      mma_commit(&sm.s_empty[b]);  // the buffer may take product t + 3
      mma_commit(&sm.v_empty[s]);
    }
  }
  mma_commit(&sm.mma_final[1]);
  mbar_wait(&sm.mma_final[1], 0, p.wait_ns);
}

template <bool kWindow>
__global__ void __launch_bounds__(kF128Threads, 1) attn_fwd128_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  Fwd128Smem& sm = *reinterpret_cast<Fwd128Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kF128QStages; ++i) {
      mbar_init(&sm.q_loaded[i], 1);
      mbar_init(&sm.q_full[i], 128);
      mbar_init(&sm.q_empty[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&sm.s_full[0][i], 1);
      mbar_init(&sm.s_full[1][i], 1);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.s_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sm.o_done[i], 1);
    for (int s = 0; s < kF128Stages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.mma_final[0], 1);
    mbar_init(&sm.mma_final[1], 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int wg = warp >> 2;
  if (wg == 1) {
    reg_alloc<kF128RegsSoftmax>();
    fwd_softmax_role<kWindow, 128, Fwd128Smem>(p, sm, tmem, 0);
  } else if (wg == 0) {
    reg_dealloc<kF128RegsRope>();
    fwd128_rope_role(p, sm);
  } else {
    reg_dealloc<kF128RegsOther>();
    if (warp == 8 && lane == 0) fwd128_producer_kv_role(p, sm);
    else if (warp == 9 && lane == 0) fwd128_mma_s_role(p, sm, tmem);
    else if (warp == 10 && lane == 0) fwd128_mma_pv_role(p, sm, tmem);
    else if (warp == 11 && lane == 0) fwd128_producer_q_role(p, sm);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace gptoss
