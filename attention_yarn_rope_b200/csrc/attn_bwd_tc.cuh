// attn_bwd_tc.cuh -- dK and dV of the sink attention backward on the 5th-
// generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Rule: as attn_bwd.cuh (the derivative of GptOssAttention's forward, NeMo
// AutoModel gpt_oss.layers page, with the RoPE of gpt_oss.rope_utils): for a
// key tile of kv head g, dV = sum over the query heads h of the group and
// every query row i that sees the key of P_ij dout_i, and dK' = scale * sum
// dS_ij q'_i, dS_ij = P_ij (dP_ij - D_i), P_ij = exp(s_ij - lse_i).
//
// CTA = (128-key tile, kv head, sequence[, chunk of its sweep]), 18 warps:
//   warps 0-15 softmax: warp w reads TMEM lanes 32 (w % 4) .. + 31 (key rows)
//              and query columns 16 (w / 4) .. + 15 of the step; per step each
//              thread reads its quarter row of S^T and dP^T from tensor memory,
//              forms P^T (bf16) and dS^T (fp16) for those 16 queries and stores
//              them back to tensor memory for the gradient products; at the
//              end warps 0-3 read and write dV, warps 4-7 dK (scale and c R^T),
//              or add them into fp32 accumulators when sweeps are split;
//   warp 16    producer: K and V tiles once (TMA), then per step the step's
//              rotated q tile (fp16) and dout tile (bf16) by TMA and its 64
//              lse and 64 D values by cp.async, kBwdTcStages ahead, all
//              completing on the stage's qd_full barrier;
//   warp 17    MMA issuer (one thread) and tensor-memory owner.
// Per step (query head h, 64-query tile), all M = 128, N = 64, K = 4 x 16:
//   S^T  = K Q^T            (SS, fp16, both K-major)
//   dP^T = V dout^T         (SS, bf16, both K-major)
//   dV  += P^T dout         (TS: P^T from tensor memory, dout read N-major)
//   dK  += dS^T Q           (TS: dS^T from tensor memory, Q read N-major)
// S^T / dP^T / P^T / dS^T have two tensor-memory sets, so step t's S^T and
// dP^T products run while the softmax warps work on step t-1; the gradient
// products of step t-1 are issued right after step t's S^T / dP^T.
// Tensor memory (512 columns): set X at 192 X: S^T [0, 64), dP^T [64, 128),
// P^T [128, 160), dS^T [160, 192); dV [384, 448), dK [448, 512).
#pragma once

#include "attn_bwd.cuh"
#include "host_util.cuh"
#include "sm100_ptx.cuh"

namespace gptoss {

constexpr int kBwdTcKeys = 128;      // keys per CTA (the M side)
constexpr int kBwdTcQ = 64;          // queries per step (the N side)
constexpr int kBwdTcStages = 6;      // q / dout buffers: loads run 5 steps ahead of their use (measured: 6 beat 4 by 0.5 %)
// 16 softmax warps: four per sub-partition, each thread 16 columns of a step
// (measured: 8 warps of 32 columns left the per-step chain -- TMEM loads,
// exponentials, stores -- unhidden, ~3300 cycles a step against ~500 of
// tensor work)
constexpr int kBwdTcSoftmax = 512;
constexpr int kBwdTcSoftWarps = kBwdTcSoftmax / 32;
constexpr int kBwdTcCols = 16;  // columns of a 64-column step per softmax thread
constexpr int kBwdTcThreads = kBwdTcSoftmax + 64;  // + producer warp, MMA warp
// steps of one CTA when sweeps are split (measured on full causal S = 8192,
// whose longest sweep has 1024 steps: 64 -> 7.24 ms, 128 -> 7.05, 192 -> 6.99,
// 256 -> 7.01, 512 -> 7.07; fewer chunks add fewer fp32 partials, more leave
// the longest CTAs running alone)
constexpr int kBwdTcChunkIt = 192;
constexpr uint32_t kBwdTcTmemCols = 512;
constexpr uint32_t kColSet = 192, kColDP = 64, kColP = 128, kColDS = 160, kColDV = 384, kColDK = 448;

struct __align__(1024) BwdTcSmem {
  uint8_t k[kBwdTcKeys * 128];                 // rotated K tile (fp16), 128B-swizzled rows
  uint8_t v[kBwdTcKeys * 128];                 // V tile (bf16)
  uint8_t q[kBwdTcStages][kBwdTcQ * 128];      // rotated q tiles (fp16)
  uint8_t dout[kBwdTcStages][kBwdTcQ * 128];   // dout tiles (bf16)
  float lsd[kBwdTcStages][2 * kBwdTcQ];        // per stage: lse log2(e) [0, 64) and D [64, 128) of its queries
  uint64_t kv_full;
  uint64_t qd_full[kBwdTcStages], qd_empty[kBwdTcStages];
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
};

// 32 lanes x 16 consecutive 32-bit columns (thread i reads lane base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns (thread i writes lane base + i).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns (thread i writes lane base + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have completed,
// without adding to the barrier's expected count (it was initialised with
// one arrival per thread that does this).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// A row of dK or dQ in tensor memory (features [0, 32) in a, [32, 64) in
// bb) scaled and taken back through RoPE with R rotary pairs (rope_t_pair),
// as bf16 pairs: lo = features [0, 32), hi = [32, 64).
template <int R>
__device__ __forceinline__ void rope_t_row(const uint32_t (&a)[32], const uint32_t (&bb)[32], const float2* cs,
                                           float scale, uint32_t (&lo)[16], uint32_t (&hi)[16]) {
  auto g = [&](int f) { return __uint_as_float(f < 32 ? a[f] : bb[f - 32]) * scale; };
  auto put = [&](int w, uint32_t v) {  // output word w: features 2w, 2w + 1
    if (w < 16) lo[w] = v;
    else hi[w - 16] = v;
  };
#pragma unroll
  for (int j = 0; j < R; j += 2) {  // pairs j, j + 1 and their partners j + R, j + R + 1
    float xr[2], yr[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) rope_t_pair(g(j + u), g(j + u + R), __ldg(cs + j + u), xr[u], yr[u]);
    put(j / 2, pack_bf16(xr[0], xr[1]));
    put((j + R) / 2, pack_bf16(yr[0], yr[1]));
  }
#pragma unroll
  for (int f = 2 * R; f < 64; f += 2) put(f / 2, pack_bf16(g(f), g(f + 1)));  // past the rotary features
}

// rope_t_row for the call's rotary pairs (a multiple of 8: rotary_dim is a
// multiple of 16).
__device__ __forceinline__ void rope_t_row_r(int R, const uint32_t (&a)[32], const uint32_t (&bb)[32],
                                             const float2* cs, float scale, uint32_t (&lo)[16], uint32_t (&hi)[16]) {
  switch (R) {
    case 8: rope_t_row<8>(a, bb, cs, scale, lo, hi); break;
    case 16: rope_t_row<16>(a, bb, cs, scale, lo, hi); break;
    case 24: rope_t_row<24>(a, bb, cs, scale, lo, hi); break;
    default: rope_t_row<32>(a, bb, cs, scale, lo, hi); break;
  }
}

// fp16 A and B with B read N-major (the q tile in dK += dS^T Q).
__host__ __device__ constexpr uint32_t idesc_f16_f32_bmn(int M, int N) { return idesc_f16_f32(M, N) | (1u << 16); }

// Bits [max(lo, 0), min(hi, 15)] of a 16-bit mask (empty when lo > hi).
__device__ __forceinline__ uint32_t col_mask16(int lo, int hi) {
  const uint32_t upto = hi >= 15 ? 0xffffu : (hi < 0 ? 0u : (2u << hi) - 1u);
  const uint32_t from = lo <= 0 ? 0xffffu : (lo > 15 ? 0u : (0xffffu << lo) & 0xffffu);
  return upto & from;
}

// P^T (bf16) and dS^T = P^T (dP^T - D) (fp16) for 16 query columns of one key
// row: P = 2^(s scale log2(e) - lse log2(e)), zero where bit c of `vis` is
// clear (kMasked).  lse2 / dsum: the columns' lse in log2 units and D.
template <bool kMasked>
__device__ __forceinline__ void bwd_p_ds(const uint32_t (&sv)[16], const uint32_t (&dv)[16], const float4 (&l4s)[4],
                                         const float4 (&d4s)[4], float sl, uint32_t vis, uint32_t (&pk)[8],
                                         uint32_t (&dk)[8]) {
#pragma unroll
  for (int e = 0; e < 16; e += 4) {
    const float4 l4 = l4s[e / 4];
    const float4 d4 = d4s[e / 4];
    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
    const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
    float pv[4], ds[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      pv[u] = ex2_approx(fmaf(__uint_as_float(sv[e + u]), sl, -lv[u]));
      if (kMasked) pv[u] = (vis >> (e + u)) & 1u ? pv[u] : 0.f;
      ds[u] = pv[u] * (__uint_as_float(dv[e + u]) - dd[u]);
    }
    pk[e / 2] = pack_bf16(pv[0], pv[1]);
    pk[e / 2 + 1] = pack_bf16(pv[2], pv[3]);
    dk[e / 2] = pack_f16(ds[0], ds[1]);
    dk[e / 2 + 1] = pack_f16(ds[2], ds[3]);
  }
}

// The CTA's sweep: steps [it0, it1) over (query head of the group, query
// tile), query tiles [qt0, qt0 + n_qt) of the sequence.
struct BwdTcWork {
  int b, kt, k0, qt0, n_qt, it0, it1;
  BwdSeq sq;
};

template <bool kSplit>
__device__ __forceinline__ bool bwd_tc_work(const BwdParams& p, BwdTcWork& w) {
  w.kt = blockIdx.x;
  w.b = kSplit ? static_cast<int>(blockIdx.z) / p.max_chunks : static_cast<int>(blockIdx.z);
  const int chunk = kSplit ? static_cast<int>(blockIdx.z) - w.b * p.max_chunks : 0;
  w.sq = bwd_seq(p, w.b);
  w.k0 = w.kt * kBwdTcKeys;
  if (w.k0 >= w.sq.L) return false;
  const int L = w.sq.L, W = p.window;
  // queries that see a key of the tile: [k0, last row that sees key k0 + 127]
  const int q_last = W > 0 ? min(L - 1, w.k0 + kBwdTcKeys - 1 + W - 1) : L - 1;
  w.qt0 = w.k0 / kBwdTcQ;
  w.n_qt = q_last / kBwdTcQ - w.qt0 + 1;
  const int n_it = p.G * w.n_qt;
  w.it0 = chunk * kBwdTcChunkIt;
  if (w.it0 >= n_it) return false;
  w.it1 = kSplit ? min(n_it, w.it0 + kBwdTcChunkIt) : n_it;
  return true;
}

// The whole producer warp runs this: lane 0 issues the TMA copies, every lane
// copies 4 of the step's 128 lse / D values.
__device__ __forceinline__ void bwd_tc_producer(const BwdParams& p, BwdTcSmem& sm, const BwdTcWork& w, int g) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    tma_prefetch_desc(&p.tmap_k);
    tma_prefetch_desc(&p.tmap_v);
    tma_prefetch_desc(&p.tmap_q);
    tma_prefetch_desc(&p.tmap_do);
  }
  const bool thd = p.cu_seqlens != nullptr;
  const int row0 = thd ? static_cast<int>(w.sq.tok0) : 0;  // token row of the sequence's first token
  const int bc = thd ? 0 : w.b;
  const int L = w.sq.L;
  if (lane == 0) {
    // the 128-row K and V tiles as two 64-row boxes each (every map's box is
    // 64 rows; the swizzle repeats every 8 rows, so the halves line up)
    mbar_arrive_expect_tx(&sm.kv_full, 2 * kBwdTcKeys * 128);
    for (int hf = 0; hf < 2; ++hf) {
      tma_load_4d(sm.k + hf * 64 * 128, &p.tmap_k, &sm.kv_full, 0, g, row0 + w.k0 + 64 * hf, bc);
      tma_load_4d(sm.v + hf * 64 * 128, &p.tmap_v, &sm.kv_full, 0, g, row0 + w.k0 + 64 * hf, bc);
    }
  }
  int issued = 0;
  for (int it = w.it0; it < w.it1; ++it, ++issued) {
    const int t = it - w.it0, s = t % kBwdTcStages;
    if (!mbar_wait_warp(&sm.qd_empty[s], ((t / kBwdTcStages) & 1) ^ 1, p.wait_ns)) break;
    const int h = g * p.G + it / w.n_qt;
    const int i0 = (w.qt0 + it % w.n_qt) * kBwdTcQ;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.qd_full[s], 2 * kBwdTcQ * 128);
      tma_load_4d(sm.q[s], &p.tmap_q, &sm.qd_full[s], 0, h, row0 + i0, bc);
      tma_load_4d(sm.dout[s], &p.tmap_do, &sm.qd_full[s], 0, h, row0 + i0, bc);
    }
    // slots 4 lane .. 4 lane + 3: lse log2(e) of queries [0, 64) (scaled once
    // by the preprocess kernel), D of [64, 128); a query past the sequence
    // copies the last row's (finite, masked anyway)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int slot = 4 * lane + u;
      const int i = min(i0 + (slot & (kBwdTcQ - 1)), L - 1);
      const int64_t ri = bwd_row_index(p, w.b, h, i, w.sq.tok0);
      cp_async4(smem_u32(&sm.lsd[s][slot]), (slot < kBwdTcQ ? p.lse2 : p.dsum) + ri);
    }
    cp_async_mbar_arrive_noinc(&sm.qd_full[s]);
  }
  // every issued copy must land before the CTA may exit
  mbar_wait(&sm.kv_full, 0, p.wait_ns);
  for (int t = issued > kBwdTcStages ? issued - kBwdTcStages : 0; t < issued; ++t)
    mbar_wait(&sm.qd_full[t % kBwdTcStages], (t / kBwdTcStages) & 1, p.wait_ns);
}

__device__ __forceinline__ void bwd_tc_mma(const BwdParams& p, BwdTcSmem& sm, const BwdTcWork& w, uint32_t tmem) {
  constexpr uint32_t idesc_s = idesc_f16_f32(128, 64);          // K (fp16) x Q^T
  constexpr uint32_t idesc_dp = idesc_bf16_f32(128, 64, false);  // V (bf16) x dout^T
  constexpr uint32_t idesc_dv = idesc_bf16_f32(128, 64, true);   // P^T (TMEM) x dout, dout N-major
  constexpr uint32_t idesc_dk = idesc_f16_f32_bmn(128, 64);      // dS^T (TMEM) x Q, Q N-major
  const int n = w.it1 - w.it0;
  const uint64_t kdesc = sw128_desc(smem_u32(sm.k));
  const uint64_t vdesc = sw128_desc(smem_u32(sm.v));
  bool ok = mbar_wait(&sm.kv_full, 0, p.wait_ns);
  // dV += P^T(u) dout(u), dK += dS^T(u) Q(u) for step u, once its P^T / dS^T exist
  auto grads = [&](int u) -> bool {
    const uint32_t X = u & 1, s = u % kBwdTcStages;
    if (!mbar_wait(&sm.p_full[X], (u >> 1) & 1, p.wait_ns)) return false;
    tc_fence_after();
    const uint64_t odesc = sw128_desc(smem_u32(sm.dout[s]));
    const uint64_t qdesc = sw128_desc(smem_u32(sm.q[s]));
    const uint32_t set = tmem + X * kColSet;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t acc = (u == 0 && kk == 0) ? 0u : 1u;
      mma_ts(tmem + kColDV, set + kColP + kk * 8, odesc + static_cast<uint64_t>(kk * 128), idesc_dv, acc);
      mma_ts(tmem + kColDK, set + kColDS + kk * 8, qdesc + static_cast<uint64_t>(kk * 128), idesc_dk, acc);
    }
    mma_commit(&sm.qd_empty[s]);  // the step's q / dout tiles are free once these complete
    return true;
  };
  for (int t = 0; t < n && ok; ++t) {
    const uint32_t X = t & 1, s = t % kBwdTcStages;
    if (!mbar_wait(&sm.qd_full[s], (t / kBwdTcStages) & 1, p.wait_ns)) { ok = false; break; }
    if (t >= 2 && !mbar_wait(&sm.s_free[X], ((t - 2) >> 1) & 1, p.wait_ns)) { ok = false; break; }
    tc_fence_after();
    const uint64_t qdesc = sw128_desc(smem_u32(sm.q[s]));
    const uint64_t odesc = sw128_desc(smem_u32(sm.dout[s]));
    const uint32_t set = tmem + X * kColSet;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(set, kdesc + static_cast<uint64_t>(kk * 2), qdesc + static_cast<uint64_t>(kk * 2), idesc_s,
             kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(set + kColDP, vdesc + static_cast<uint64_t>(kk * 2), odesc + static_cast<uint64_t>(kk * 2), idesc_dp,
             kk > 0 ? 1u : 0u);
    mma_commit(&sm.s_full[X]);
    if (t >= 1 && !grads(t - 1)) ok = false;
  }
  if (ok && n > 0) grads(n - 1);
  // dV and dK are final once every product above has completed
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, p.wait_ns);
}

template <bool kSplit>
__device__ __forceinline__ void bwd_tc_softmax(const BwdParams& p, BwdTcSmem& sm, const BwdTcWork& w, int g,
                                               uint32_t tmem) {
  const int tid = threadIdx.x;         // 0 .. 511
  const int wq = (tid >> 5) & 3;       // TMEM lane quarter
  const int ch = tid >> 7;             // query-column quarter of the step
  const int r = wq * 32 + (tid & 31);  // key row of the tile = TMEM lane
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int L = w.sq.L, W = p.window;
  const int j = w.k0 + r;              // this thread's key
  const bool j_ok = j < L;
  const float sl = p.scale_log2;
  const int n = w.it1 - w.it0;
  for (int t = 0; t < n; ++t) {
    const int it = w.it0 + t;
    const int i0 = (w.qt0 + it % w.n_qt) * kBwdTcQ + ch * kBwdTcCols;  // this thread's first query column
    const uint32_t X = t & 1;
    const int stg = t % kBwdTcStages;
    // the step's lse / D landed with its tiles (cp.async on qd_full); they
    // stay until this step's gradient products free the stage (qd_empty),
    // which follows this thread's p_full arrival below
    if (!mbar_wait_warp(&sm.qd_full[stg], (t / kBwdTcStages) & 1, p.wait_ns)) return;
    // the step's lse / D columns, read while S^T / dP^T are still in flight
    float4 l4s[4], d4s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      l4s[e] = *reinterpret_cast<const float4*>(&sm.lsd[stg][ch * kBwdTcCols + 4 * e]);
      d4s[e] = *reinterpret_cast<const float4*>(&sm.lsd[stg][kBwdTcQ + ch * kBwdTcCols + 4 * e]);
    }
    if (!mbar_wait_warp(&sm.s_full[X], (t >> 1) & 1, p.wait_ns)) return;
    tc_fence_after();
    const uint32_t set = lane_base + X * kColSet;
    uint32_t sv[kBwdTcCols], dv[kBwdTcCols];
    tmem_ld16(set + ch * kBwdTcCols, sv);
    tmem_ld16(set + kColDP + ch * kBwdTcCols, dv);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&sm.s_free[X]);  // S^T / dP^T of set X may be overwritten
    // every pair of this warp's 32 keys x 16 queries visible: no mask
    const int jw = w.k0 + wq * 32;
    const bool all_vis = jw + 31 <= i0 && i0 + kBwdTcCols - 1 < L && jw + 31 < L &&
                         (W == 0 || i0 + kBwdTcCols - 1 - jw < W);
    uint32_t pk[kBwdTcCols / 2], dk[kBwdTcCols / 2];
    if (all_vis) {
      bwd_p_ds<false>(sv, dv, l4s, d4s, sl, 0u, pk, dk);
    } else {  // this key's visible queries i0 + c: c in [j - i0, min(L - 1, j + W - 1) - i0]
      const int hi = (W > 0 ? min(L - 1, j + W - 1) : L - 1) - i0;
      bwd_p_ds<true>(sv, dv, l4s, d4s, sl, j_ok ? col_mask16(j - i0, hi) : 0u, pk, dk);
    }
    // P^T / dS^T of set X were last read by step t-2's gradient products,
    // which completed before step t's S^T (s_full covers all earlier products)
    tmem_st8(set + kColP + ch * (kBwdTcCols / 2), pk);
    tmem_st8(set + kColDS + ch * (kBwdTcCols / 2), dk);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&sm.p_full[X]);
  }
  // ---- epilogue: warps 0-3 write dV, warps 4-7 dK, one key row per thread ----
  if (ch >= 2) return;  // warp-uniform: warps 8-15 have no epilogue
  if (!mbar_wait_warp(&sm.mma_done, 0, p.wait_ns)) return;
  tc_fence_after();
  const int which = ch;  // 0: dV, 1: dK
  const int64_t tok = w.sq.tok0 + j;
  const int64_t row = (tok * p.Hkv + g) * kHeadDim;
  uint32_t a[32], bb[32];
  const uint32_t col = which == 0 ? kColDV : kColDK;
  tmem_ld32(lane_base + col, a);        // features [0, 32)
  tmem_ld32(lane_base + col + 32, bb);  // features [32, 64)
  tmem_wait_ld();
  if (!j_ok) return;
  if (kSplit) {
    float* acc = (which == 0 ? p.dv_acc : p.dk_acc) + row;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      atomicAdd(reinterpret_cast<float2*>(acc + e), make_float2(__uint_as_float(a[e]), __uint_as_float(a[e + 1])));
      atomicAdd(reinterpret_cast<float2*>(acc + 32 + e),
                make_float2(__uint_as_float(bb[e]), __uint_as_float(bb[e + 1])));
    }
    return;
  }
  __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + row;
  uint32_t lo[16], hi[16];
  if (which == 0) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      lo[e] = pack_bf16(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
      hi[e] = pack_bf16(__uint_as_float(bb[2 * e]), __uint_as_float(bb[2 * e + 1]));
    }
  } else {  // scale, then c R^T
    rope_t_row_r(p.R, a, bb, p.cs + tok * kPairs, p.scale, lo, hi);
  }
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    reinterpret_cast<uint4*>(dst)[q4] = make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
    reinterpret_cast<uint4*>(dst + 32)[q4] = make_uint4(hi[4 * q4], hi[4 * q4 + 1], hi[4 * q4 + 2], hi[4 * q4 + 3]);
  }
}

template <bool kSplit>
__global__ void __launch_bounds__(kBwdTcThreads, 1) attn_bwd_dkdv_tc_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  BwdTcSmem& sm = *reinterpret_cast<BwdTcSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdTcWork w;
  if (!bwd_tc_work<kSplit>(p, w)) return;  // uniform over the CTA, before any barrier
  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < kBwdTcStages; ++s) {
      mbar_init(&sm.qd_full[s], 1 + 32);  // the TMA arrival + one cp.async arrival per producer lane
      mbar_init(&sm.qd_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.s_free[x], kBwdTcSoftmax);
      mbar_init(&sm.p_full[x], kBwdTcSoftmax);
    }
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kBwdTcSoftWarps + 1) {
    tmem_alloc(&sm.tmem_base, kBwdTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < kBwdTcSoftWarps) bwd_tc_softmax<kSplit>(p, sm, w, g, tmem);
  else if (warp == kBwdTcSoftWarps) bwd_tc_producer(p, sm, w, g);
  else if (warp == kBwdTcSoftWarps + 1 && lane == 0) bwd_tc_mma(p, sm, w, tmem);
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdTcSoftWarps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTcTmemCols);
  }
}

// ============================================================================
// dQ on the tensor cores.  CTA = (128-query tile, head, sequence), 18 warps:
// 16 softmax warps (TMEM lanes 32 (w % 4) .. = query rows, key columns
// 16 (w / 4) .. of the step), a TMA producer (Q and dout tiles once, then each
// step's 64-key K and V tiles, kBwdTcStages ahead), an MMA issuer.  Per step:
//   S  = Q K^T, dP = dout V^T   (SS, K-major; M = 128 queries, N = 64 keys)
//   dS = P (dP - D) -> tensor memory (fp16), P = exp(S scale - lse)
//   dQ += dS K                  (TS: dS from tensor memory, K read N-major)
// lse and D belong to the thread's own row, so they are loaded once.  TMEM:
// set X at 192 X: S [0, 64), dP [64, 128), dS [128, 160); dQ [384, 448).
// ============================================================================
constexpr uint32_t kColDQ = 384;

struct __align__(1024) BwdTcQSmem {
  uint8_t q[128 * 128];                        // rotated Q tile (fp16), 128B-swizzled rows
  uint8_t dout[128 * 128];                     // dout tile (bf16)
  uint8_t k[kBwdTcStages][kBwdTcQ * 128];      // rotated K tiles (fp16), 64 keys
  uint8_t v[kBwdTcStages][kBwdTcQ * 128];      // V tiles (bf16)
  uint64_t qd_full;
  uint64_t kv_full[kBwdTcStages], kv_empty[kBwdTcStages];
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
};

struct BwdTcQWork {
  int b, h, q0, kt0, n;  // query tile start, first key tile (64 keys), steps
  BwdSeq sq;
};

__device__ __forceinline__ bool bwd_tcq_work(const BwdParams& p, BwdTcQWork& w) {
  const int n_qt = (p.S + 127) / 128;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x);  // the longest sweeps start first
  w.h = blockIdx.y;
  w.b = blockIdx.z;
  w.sq = bwd_seq(p, w.b);
  w.q0 = qt * 128;
  if (w.q0 >= w.sq.L) return false;
  const int L = w.sq.L, W = p.window;
  const int j_first = W > 0 ? max(0, w.q0 - W + 1) : 0;
  const int j_last = min(L - 1, w.q0 + 127);
  w.kt0 = j_first / kBwdTcQ;
  w.n = j_last / kBwdTcQ - w.kt0 + 1;
  return true;
}

__device__ __forceinline__ void bwd_tcq_producer(const BwdParams& p, BwdTcQSmem& sm, const BwdTcQWork& w) {
  tma_prefetch_desc(&p.tmap_k);
  tma_prefetch_desc(&p.tmap_v);
  tma_prefetch_desc(&p.tmap_q);
  tma_prefetch_desc(&p.tmap_do);
  const bool thd = p.cu_seqlens != nullptr;
  const int row0 = thd ? static_cast<int>(w.sq.tok0) : 0;
  const int bc = thd ? 0 : w.b;
  const int g = w.h / p.G;
  mbar_arrive_expect_tx(&sm.qd_full, 2 * 128 * 128);
  for (int hf = 0; hf < 2; ++hf) {
    tma_load_4d(sm.q + hf * 64 * 128, &p.tmap_q, &sm.qd_full, 0, w.h, row0 + w.q0 + 64 * hf, bc);
    tma_load_4d(sm.dout + hf * 64 * 128, &p.tmap_do, &sm.qd_full, 0, w.h, row0 + w.q0 + 64 * hf, bc);
  }
  int issued = 0;
  for (int t = 0; t < w.n; ++t, ++issued) {
    const int s = t % kBwdTcStages;
    if (!mbar_wait(&sm.kv_empty[s], ((t / kBwdTcStages) & 1) ^ 1, p.wait_ns)) break;
    const int j0 = (w.kt0 + t) * kBwdTcQ;
    mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kBwdTcQ * 128);
    tma_load_4d(sm.k[s], &p.tmap_k, &sm.kv_full[s], 0, g, row0 + j0, bc);
    tma_load_4d(sm.v[s], &p.tmap_v, &sm.kv_full[s], 0, g, row0 + j0, bc);
  }
  // every issued copy must land before the CTA may exit
  mbar_wait(&sm.qd_full, 0, p.wait_ns);
  for (int t = issued > kBwdTcStages ? issued - kBwdTcStages : 0; t < issued; ++t)
    mbar_wait(&sm.kv_full[t % kBwdTcStages], (t / kBwdTcStages) & 1, p.wait_ns);
}

__device__ __forceinline__ void bwd_tcq_mma(const BwdParams& p, BwdTcQSmem& sm, const BwdTcQWork& w, uint32_t tmem) {
  constexpr uint32_t idesc_s = idesc_f16_f32(128, 64);          // Q (fp16) x K^T
  constexpr uint32_t idesc_dp = idesc_bf16_f32(128, 64, false);  // dout (bf16) x V^T
  constexpr uint32_t idesc_dq = idesc_f16_f32_bmn(128, 64);      // dS (TMEM) x K, K N-major
  const uint64_t qdesc = sw128_desc(smem_u32(sm.q));
  const uint64_t odesc = sw128_desc(smem_u32(sm.dout));
  bool ok = mbar_wait(&sm.qd_full, 0, p.wait_ns);
  auto grads = [&](int u) -> bool {  // dQ += dS(u) K(u)
    const uint32_t X = u & 1, s = u % kBwdTcStages;
    if (!mbar_wait(&sm.p_full[X], (u >> 1) & 1, p.wait_ns)) return false;
    tc_fence_after();
    const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s]));
    const uint32_t set = tmem + X * kColSet;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(tmem + kColDQ, set + kColP + kk * 8, kdesc + static_cast<uint64_t>(kk * 128), idesc_dq,
             (u == 0 && kk == 0) ? 0u : 1u);
    mma_commit(&sm.kv_empty[s]);  // the step's K / V tiles are free once these complete
    return true;
  };
  for (int t = 0; t < w.n && ok; ++t) {
    const uint32_t X = t & 1, s = t % kBwdTcStages;
    if (!mbar_wait(&sm.kv_full[s], (t / kBwdTcStages) & 1, p.wait_ns)) { ok = false; break; }
    if (t >= 2 && !mbar_wait(&sm.s_free[X], ((t - 2) >> 1) & 1, p.wait_ns)) { ok = false; break; }
    tc_fence_after();
    const uint64_t kdesc = sw128_desc(smem_u32(sm.k[s]));
    const uint64_t vdesc = sw128_desc(smem_u32(sm.v[s]));
    const uint32_t set = tmem + X * kColSet;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(set, qdesc + static_cast<uint64_t>(kk * 2), kdesc + static_cast<uint64_t>(kk * 2), idesc_s,
             kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(set + kColDP, odesc + static_cast<uint64_t>(kk * 2), vdesc + static_cast<uint64_t>(kk * 2), idesc_dp,
             kk > 0 ? 1u : 0u);
    mma_commit(&sm.s_full[X]);
    if (t >= 1 && !grads(t - 1)) ok = false;
  }
  if (ok && w.n > 0) grads(w.n - 1);
  mma_commit(&sm.mma_done);
  mbar_wait(&sm.mma_done, 0, p.wait_ns);
}

template <int R>
__device__ __forceinline__ void bwd_tcq_softmax(const BwdParams& p, BwdTcQSmem& sm, const BwdTcQWork& w,
                                                uint32_t tmem) {
  const int tid = threadIdx.x;         // 0 .. 511
  const int wq = (tid >> 5) & 3;       // TMEM lane quarter
  const int ch = tid >> 7;             // key-column quarter of the step
  const int r = wq * 32 + (tid & 31);  // query row of the tile = TMEM lane
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int L = w.sq.L, W = p.window;
  const int i = w.q0 + r;              // this thread's query
  const bool i_ok = i < L;
  const float sl = p.scale_log2;
  float lse2 = 0.f, dd = 0.f;
  if (i_ok) {
    const int64_t ri = bwd_row_index(p, w.b, w.h, i, w.sq.tok0);
    lse2 = __ldg(p.lse + ri) * kLog2e;
    dd = __ldg(p.dsum + ri);
  }
  const int iw = w.q0 + wq * 32;  // this warp's first query row
  for (int t = 0; t < w.n; ++t) {
    const uint32_t X = t & 1;
    const int j0 = (w.kt0 + t) * kBwdTcQ + ch * kBwdTcCols;  // this thread's first key column
    if (!mbar_wait_warp(&sm.s_full[X], (t >> 1) & 1, p.wait_ns)) return;
    tc_fence_after();
    const uint32_t set = lane_base + X * kColSet;
    uint32_t sv[kBwdTcCols], dv[kBwdTcCols];
    tmem_ld16(set + ch * kBwdTcCols, sv);
    tmem_ld16(set + kColDP + ch * kBwdTcCols, dv);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(&sm.s_free[X]);  // S / dP of set X may be overwritten
    // every pair of this warp's 32 queries x 16 keys visible: no mask
    const bool all_vis = j0 + kBwdTcCols - 1 <= iw && iw + 31 < L && (W == 0 || iw + 31 - j0 < W);
    // else this query's visible keys j0 + c: c in [i - W + 1 - j0, i - j0]
    const uint32_t vis = all_vis ? 0xffffu : (i_ok ? col_mask16(W > 0 ? i - W + 1 - j0 : 0, i - j0) : 0u);
    uint32_t dk[kBwdTcCols / 2];
#pragma unroll
    for (int e = 0; e < kBwdTcCols; e += 2) {
      float ds[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float pv = ex2_approx(fmaf(__uint_as_float(sv[e + u]), sl, -lse2));
        pv = (vis >> (e + u)) & 1u ? pv : 0.f;
        ds[u] = pv * (__uint_as_float(dv[e + u]) - dd);
      }
      dk[e / 2] = pack_f16(ds[0], ds[1]);
    }
    // dS of set X was last read by step t-2's dQ product, which completed
    // before step t's S (s_full covers all earlier products)
    tmem_st8(set + kColP + ch * (kBwdTcCols / 2), dk);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&sm.p_full[X]);
  }
  // ---- epilogue: warps 0-3 write this query row of dq (scale, c R^T) ----
  if (ch != 0) return;  // warp-uniform
  if (!mbar_wait_warp(&sm.mma_done, 0, p.wait_ns)) return;
  tc_fence_after();
  uint32_t a[32], bb[32];
  tmem_ld32(lane_base + kColDQ, a);        // features [0, 32)
  tmem_ld32(lane_base + kColDQ + 32, bb);  // features [32, 64)
  tmem_wait_ld();
  if (!i_ok) return;
  const int64_t tok = w.sq.tok0 + i;
  __nv_bfloat16* dst = p.dq + (tok * p.Hq + w.h) * kHeadDim;
  uint32_t lo[16], hi[16];
  rope_t_row<R>(a, bb, p.cs + tok * kPairs, p.scale, lo, hi);
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    reinterpret_cast<uint4*>(dst)[q4] = make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
    reinterpret_cast<uint4*>(dst + 32)[q4] = make_uint4(hi[4 * q4], hi[4 * q4 + 1], hi[4 * q4 + 2], hi[4 * q4 + 3]);
  }
}

// R: the call's rotary pairs (p.R), a template parameter as for
// attn_bwd_dq_kernel (measured: a runtime switch cost full causal 0.7 %).
template <int R>
__global__ void __launch_bounds__(kBwdTcThreads, 1) attn_bwd_dq_tc_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  BwdTcQSmem& sm = *reinterpret_cast<BwdTcQSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  BwdTcQWork w;
  if (!bwd_tcq_work(p, w)) return;  // uniform over the CTA, before any barrier
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.qd_full, 1);
    for (int s = 0; s < kBwdTcStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.s_free[x], kBwdTcSoftmax);
      mbar_init(&sm.p_full[x], kBwdTcSoftmax);
    }
    mbar_init(&sm.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == kBwdTcSoftWarps + 1) {
    tmem_alloc(&sm.tmem_base, kBwdTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp < kBwdTcSoftWarps) bwd_tcq_softmax<R>(p, sm, w, tmem);
  else if (warp == kBwdTcSoftWarps && lane == 0) bwd_tcq_producer(p, sm, w);
  else if (warp == kBwdTcSoftWarps + 1 && lane == 0) bwd_tcq_mma(p, sm, w, tmem);
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdTcSoftWarps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kBwdTcTmemCols);
  }
}

}  // namespace gptoss
