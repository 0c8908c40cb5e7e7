// fwd_pipeline.cuh -- TMA producer, tcgen05 MMA issuers and the prefill
// kernel itself (gptoss_attn_fwd).
//
// Products (each consumer is signalled by tcgen05.commit on an mbarrier):
//   S_X(t) = Q_X K(t)^T   (SS, M128 N128, 4 x K16)
//   O_X += P_X(t) V(t)    (TS: P from TMEM, V from shared memory read N-major,
//                          M128 N64, 8 x K16)
#pragma once

#include "fwd_common.cuh"
#include "fwd_rope.cuh"
#include "fwd_softmax.cuh"

namespace gptoss {

// =============================== TMA producers ===============================
// K / V tiles of every unit, in unit order, into the 4-stage ring.
__device__ __forceinline__ void fwd_producer_kv_role(const FwdParams& p, FwdSmem& sm) {
  tma_prefetch_desc(&p.tmap_k);
  tma_prefetch_desc(&p.tmap_v);
  const bool thd = p.cu_seqlens != nullptr;
  uint32_t kv_it = 0, k_issued = 0, v_issued = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int tok0 = thd ? wu.seq_start : 0;
    const int bc = thd ? 0 : wu.b;
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
  for (uint32_t it = k_issued > kFwdStages ? k_issued - kFwdStages : 0; it < k_issued; ++it)
    mbar_wait(&sm.k_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
  for (uint32_t it = v_issued > kFwdStages ? v_issued - kFwdStages : 0; it < v_issued; ++it)
    mbar_wait(&sm.v_full[it % kFwdStages], (it / kFwdStages) & 1, p.wait_ns);
}

// The two raw Q tiles of every unit into the 3-stage Q ring.  Its own warp,
// so a Q load never queues behind a K / V stage that is still in use: with
// two-tile units (128-key window) the Q of a unit must be requested two
// units ahead to hide the HBM latency.
__device__ __forceinline__ void fwd_producer_q_role(const FwdParams& p, FwdSmem& sm) {
  tma_prefetch_desc(&p.tmap_q);
  const bool thd = p.cu_seqlens != nullptr;
  uint32_t i = 0;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qs = i % kFwdQStages;
    if (!mbar_wait(&sm.q_empty[qs], ((i / kFwdQStages) & 1) ^ 1, p.wait_ns)) break;
    mbar_arrive_expect_tx(&sm.q_loaded[qs], 2 * kFwdTileBytes);
    const int tok = (thd ? wu.seq_start : 0) + wu.q0;
    const int bc = thd ? 0 : wu.b;
    tma_load_4d(sm.q[qs][0], &p.tmap_q, &sm.q_loaded[qs], 0, wu.h0, tok, bc);
    tma_load_4d(sm.q[qs][1], &p.tmap_q, &sm.q_loaded[qs], 0, wu.h1, tok, bc);
    ++i;
  }
  // the copies of the last stages must land before the CTA exits
  for (uint32_t it = i > kFwdQStages ? i - kFwdQStages : 0; it < i; ++it)
    mbar_wait(&sm.q_loaded[it % kFwdQStages], (it / kFwdQStages) & 1, p.wait_ns);
}

// ================================ MMA issuers ================================
// Two threads issue the tensor-core work.  A tcgen05.mma blocks its issuing
// thread until the tensor core takes it, and a product's completion reaches
// its consumer roughly 450 cycles after issue; with one issuer, the next
// QK^T would queue behind the previous tile's P V issue and wait for the
// softmax's P.  Split, QK^T depends only on the softmax having read S (early
// in each tile) and P V only on P: each is issued as soon as its inputs exist.
// tcgen05.commit tracks the issuing thread's own products, so each thread
// signals its own consumers.

// S_X(t) = Q_X K(t)^T for both head slots, tile by tile.  kTri: the
// three-buffer layout, else per slot (fwd_common.cuh).
template <bool kTri>
__device__ __forceinline__ void fwd_mma_s_role(const FwdParams& p, FwdSmem& sm, uint32_t tmem) {
  // Q (rotated or converted by the rope warps) and K (from the workspace) are fp16
  constexpr uint32_t idesc_s = idesc_f16_f32(128, 128);
  uint32_t t = 0, kv_it = 0, i = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    const int qb = i % kFwdQStages;
    if (!mbar_wait(&sm.q_full[qb], (i / kFwdQStages) & 1, p.wait_ns)) break;
    for (int j = 0; j < wu.n_kt; ++j, ++t, ++kv_it) {
      const int s = kv_it % kFwdStages;
      if (!mbar_wait(&sm.k_full[s], (kv_it / kFwdStages) & 1, p.wait_ns)) { ok = false; break; }
      const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s]));
#pragma unroll 1
      for (int X = 0; X < 2; ++X) {
        uint32_t b, colS;
        if (kTri) {  // product k = 2t + X into S buffer k mod 3, once product k - 3's P V has read its P
          const uint32_t k = 2 * t + X;
          b = k % kSBufs;
          colS = b * 128;
          if (k >= kSBufs && !mbar_wait(&sm.s_empty[b], ((k / kSBufs) - 1) & 1, p.wait_ns)) { ok = false; break; }
        } else {  // slot X's own S, once its softmax has read the previous one
          b = 0;
          colS = X * 256;
          if (t > 0 && !mbar_wait(&sm.s_free[X], (t - 1) & 1, p.wait_ns)) { ok = false; break; }
        }
        tc_fence_after();
        const uint64_t qdesc = sw128_desc(smem_u32(sm.q[qb][X]));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + colS, qdesc + static_cast<uint64_t>(kk * 2), kdesc + static_cast<uint64_t>(kk * 2),
                 idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[X][b]);
      }
      if (!ok) break;
      mma_commit(&sm.k_empty[s]);
      if (j == wu.n_kt - 1) mma_commit(&sm.q_empty[qb]);
    }
    ++i;
  }
  mma_commit(&sm.mma_final[0]);
  mbar_wait(&sm.mma_final[0], 0, p.wait_ns);
}

// O_X += P_X(t) V(t) for both head slots (TS: P from TMEM, V N-major from
// shared memory); the first tile of a unit starts O from zero.
template <bool kTri>
__device__ __forceinline__ void fwd_mma_pv_role(const FwdParams& p, FwdSmem& sm, uint32_t tmem) {
  constexpr uint32_t idesc_o = idesc_f16_f32(128, 64, true);  // fp16 P (TMEM) x fp16 V (workspace)
  uint32_t t = 0, kv_it = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    Unit wu;
    if (!make_unit(p, u, wu)) continue;
    for (int j = 0; j < wu.n_kt; ++j, ++t, ++kv_it) {
      const int s = kv_it % kFwdStages;
      if (!mbar_wait(&sm.v_full[s], (kv_it / kFwdStages) & 1, p.wait_ns)) { ok = false; break; }
      const uint64_t vdesc = sw128_desc(smem_u32(sm.v[s]));
#pragma unroll 1
      for (int X = 0; X < 2; ++X) {
        const uint32_t k = 2 * t + X;
        const uint32_t b = kTri ? k % kSBufs : X;  // three-buffer: P sits over the S it came from
        if (!mbar_wait(&sm.p_full[b], (kTri ? k / kSBufs : t) & 1, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t colP = kTri ? b * 128 : X * 256 + 128, colO = kTri ? kColO + X * 64 : X * 256 + 192;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + colO, tmem + colP + kk * 8, vdesc + static_cast<uint64_t>(kk * 128), idesc_o,
                 (j == 0 && kk == 0) ? 0u : 1u);
        mma_commit(&sm.o_done[X]);
        if (kTri) mma_commit(&sm.s_empty[b]);  // the buffer may take product 2t + X + 3
      }
      if (!ok) break;
      mma_commit(&sm.v_empty[s]);
    }
  }
  mma_commit(&sm.mma_final[1]);
  mbar_wait(&sm.mma_final[1], 0, p.wait_ns);
}

// ================================== kernel ==================================
template <bool kWindow>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  FwdSmem& sm = *reinterpret_cast<FwdSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kFwdQStages; ++i) {
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.o_done[i], 1);
      mbar_init(&sm.s_free[i], 128);
    }
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.mma_final[0], 1);
    mbar_init(&sm.mma_final[1], 1);
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
  // the rope warpgroup takes the lowest warp numbers (measured: its Q
  // rotation finishes sooner there, next to two busy softmax warpgroups)
  if (wg == 1 || wg == 2) {
    reg_alloc<kRegsSoftmax>();
    fwd_softmax_role<kWindow>(p, sm, tmem, wg - 1);
  } else if (wg == 0) {
    reg_dealloc<kRegsRope>();
    fwd_rope_role(p, sm);
  } else {
    reg_dealloc<kRegsOther>();
    if (warp == 12 && lane == 0) fwd_producer_kv_role(p, sm);
    else if (warp == 13 && lane == 0) fwd_mma_s_role<!kWindow>(p, sm, tmem);
    else if (warp == 14 && lane == 0) fwd_mma_pv_role<!kWindow>(p, sm, tmem);
    else if (warp == 15 && lane == 0) fwd_producer_q_role(p, sm);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmemCols);
  }
}

}  // namespace gptoss
