// fwd_pipeline.cuh -- TMA producer, tcgen05 MMA issuer and the prefill
// kernel itself (gptoss_attn_fwd).
//
// MMA order per key tile t (one thread issues everything):
//   S_A(t) = Q_A K(t)^T, S_B(t) = Q_B K(t)^T   (SS, M128 N128, 4 x K16)
//   O_A += P_A(t-1) V(t-1), O_B += P_B(t-1) V(t-1)   (TS: P from TMEM, V from
//   shared memory read N-major, M128 N64, 8 x K16)
// so the next tile's QK^T runs while the softmax warps exponentiate.  Each
// consumer is signalled by tcgen05.commit on an mbarrier.
#pragma once

#include "fwd_common.cuh"
#include "fwd_rope.cuh"
#include "fwd_softmax.cuh"

namespace gptoss {

// =============================== TMA producer ===============================
__device__ __forceinline__ void fwd_producer_role(const FwdParams& p, FwdSmem& sm) {
  tma_prefetch_desc(&p.tmap_q);
  tma_prefetch_desc(&p.tmap_k);
  tma_prefetch_desc(&p.tmap_v);
  const bool thd = p.cu_seqlens != nullptr;
  uint32_t kv_it = 0, k_issued = 0, v_issued = 0, i = 0, q_issued = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int tok0 = thd ? wu.seq_start : 0;
    const int bc = thd ? 0 : wu.b;
    // the unit's two raw Q tiles into the free half of the Q double buffer
    const int qb = i & 1;
    if (!mbar_wait(&sm.q_empty[qb], ((i >> 1) & 1) ^ 1, p.wait_ns)) break;
    mbar_arrive_expect_tx(&sm.q_loaded[qb], 2 * kFwdTileBytes);
    tma_load_4d(sm.q[qb][0], &p.tmap_q, &sm.q_loaded[qb], 0, wu.h0, tok0 + wu.q0, bc);
    tma_load_4d(sm.q[qb][1], &p.tmap_q, &sm.q_loaded[qb], 0, wu.h1, tok0 + wu.q0, bc);
    q_issued = ++i;
    for (int j = 0; j < wu.n_kt; ++j, ++kv_it) {
      const int s = kv_it % kFwdStages;
      const uint32_t ph = ((kv_it / kFwdStages) & 1) ^ 1;
      const int key_row = tok0 + (wu.j_lo + j) * kFwdTile;
      if (!mbar_wait(&sm.k_empty[s], ph, p.wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.k_full[s], kFwdTileBytes);
      tma_load_4d(sm.k[s], &p.tmap_k, &sm.k_full[s], 0, wu.g, key_row, bc);
      k_issued = kv_it + 1;
      if (!mbar_wait(&sm.v_empty[s], ph, p.wait_ns)) { ok = false; break; }
      mbar_arrive_expect_tx(&sm.v_full[s], kFwdTileBytes);
      tma_load_4d(sm.v[s], &p.tmap_v, &sm.v_full[s], 0, wu.g, key_row, bc);
      v_issued = kv_it + 1;
    }
  }
  // the copies of the last stages must land before the CTA exits
  for (uint32_t it = q_issued > 2 ? q_issued - 2 : 0; it < q_issued; ++it)
    mbar_wait(&sm.q_loaded[it & 1], (it >> 1) & 1, p.wait_ns);
  for (uint32_t it = k_issued > kFwdStages ? k_issued - kFwdStages : 0; it < k_issued; ++it)
    mbar_wait(&sm.k_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
  for (uint32_t it = v_issued > kFwdStages ? v_issued - kFwdStages : 0; it < v_issued; ++it)
    mbar_wait(&sm.v_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
}

// ================================ MMA issuer ================================
// O_X += P_X V for the tile with running index tt whose V sits in the stage of
// kv iteration kv; `first` = the tile opens its unit (O starts from zero).
__device__ __forceinline__ bool fwd_issue_pv(const FwdParams& p, FwdSmem& sm, uint32_t tmem, uint32_t tt,
                                             uint32_t kv, bool first) {
  constexpr uint32_t idesc_o = idesc_bf16_f32(128, 64, true);
  const int s = kv % kFwdStages;
  if (!mbar_wait(&sm.v_full[s], (kv / kFwdStages) & 1, p.wait_ns)) return false;
  const uint64_t vdesc = sw128_desc(smem_u32(sm.v[s]));
#pragma unroll 1
  for (int X = 0; X < 2; ++X) {
    if (!mbar_wait(&sm.p_full[X], tt & 1, p.wait_ns)) return false;
    tc_fence_after();
    const uint32_t colP = X * 256 + 128, colO = X * 256 + 192;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tmem + colO, tmem + colP + kk * 8, vdesc + static_cast<uint64_t>(kk * 128), idesc_o,
             (first && kk == 0) ? 0u : 1u);
    mma_commit(&sm.o_done[X]);
  }
  mma_commit(&sm.v_empty[s]);
  return true;
}

__device__ __forceinline__ void fwd_mma_role(const FwdParams& p, FwdSmem& sm, uint32_t tmem) {
  // fused RoPE leaves Q and K in shared memory as fp16; pre-rotated inputs stay bf16
  const uint32_t idesc_s = p.tab.enabled ? idesc_f16_f32(128, 128) : idesc_bf16_f32(128, 128, false);
  uint32_t t = 0, kv_it = 0, i = 0;
  bool have_prev = false, prev_first = false, ok = true;
  uint32_t prev_t = 0, prev_kv = 0;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qb = i & 1;
    if (!mbar_wait(&sm.q_full[qb], (i >> 1) & 1, p.wait_ns)) { ok = false; break; }
    for (int j = 0; j < wu.n_kt && ok; ++j, ++t, ++kv_it) {
      const int s = kv_it % kFwdStages;
      if (!mbar_wait(&sm.k_ready[s], (kv_it / kFwdStages) & 1, p.wait_ns)) { ok = false; break; }
      const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s]));
#pragma unroll 1
      for (int X = 0; X < 2 && ok; ++X) {
        if (t > 0 && !mbar_wait(&sm.s_free[X], (t - 1) & 1, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint64_t qdesc = sw128_desc(smem_u32(sm.q[qb][X]));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + X * 256, qdesc + static_cast<uint64_t>(kk * 2), kdesc + static_cast<uint64_t>(kk * 2),
                 idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[X]);
      }
      if (!ok) break;
      mma_commit(&sm.k_empty[s]);
      if (j == wu.n_kt - 1) mma_commit(&sm.q_empty[qb]);
      if (have_prev && !fwd_issue_pv(p, sm, tmem, prev_t, prev_kv, prev_first)) { ok = false; break; }
      have_prev = true;
      prev_t = t;
      prev_kv = kv_it;
      prev_first = (j == 0);
      if (j == wu.n_kt - 1) {
        // close the unit now: its epilogue must not wait for the next unit's
        // first QK^T (which needs that unit's Q and K tiles to be ready)
        if (!fwd_issue_pv(p, sm, tmem, prev_t, prev_kv, prev_first)) { ok = false; break; }
        have_prev = false;
      }
    }
    ++i;
  }
  if (ok && have_prev) fwd_issue_pv(p, sm, tmem, prev_t, prev_kv, prev_first);
  // every issued MMA must finish before TMEM is released
  mma_commit(&sm.mma_final);
  mbar_wait(&sm.mma_final, 0, p.wait_ns);
}

// ================================== kernel ==================================
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  FwdSmem& sm = *reinterpret_cast<FwdSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_loaded[i], 1);
      mbar_init(&sm.q_full[i], 128);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 128);
      mbar_init(&sm.p_full[i], 128);
      mbar_init(&sm.o_done[i], 1);
    }
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_ready[s], 128);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.mma_final, 1);
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(&sm.tmem_base, kFwdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int wg = warp >> 2;
  if (wg < 2) {
    reg_alloc<kRegsSoftmax>();
    fwd_softmax_role(p, sm, tmem, wg);
  } else if (wg == 2) {
    reg_dealloc<kRegsRope>();
    fwd_rope_role(p, sm);
  } else {
    reg_dealloc<kRegsOther>();
    if (warp == 12 && lane == 0) fwd_producer_role(p, sm);
    else if (warp == 13 && lane == 0) fwd_mma_role(p, sm, tmem);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace gptoss
