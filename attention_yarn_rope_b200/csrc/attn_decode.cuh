// attn_decode.cuh -- single-token decode over a bf16 KV cache (gptoss_attn_decode).
//
// Rule: the sink attention of GptOssAttention (NeMo AutoModel gpt_oss.layers
// page: sinks, sliding_window, softmax_scale) for one new query per sequence
// at position len-1 (RoPE rule of the gpt_oss.rope_utils page), keys already
// rotated in the cache; with q_len new tokens, token i at position
// len - q_len + i sees the keys up to its own (causal).
//
// Design: the op streams the cache once, so it is HBM-bound (8 FLOP per cache
// byte at 8 q-heads per kv-head).  Split-KV: CTA (g, split, b) owns one kv
// head and a contiguous chunk of keys and computes all G = Hq/Hkv query heads
// of that group, so each cache byte is read exactly once.  A producer warp
// streams 64-key K and V tiles with TMA (128-byte swizzled rows) through a
// ring of stages; four consumer warps each take 16 keys of a stage and run
// QK^T and PV on the tensor cores with warp-level mma.sync m16n8k16 (query
// heads as the 16-row M side), an online softmax per head with quad shuffles,
// and fp32 accumulators in registers.  The CTA writes an unnormalised partial
// (m, l, O) per head; a second kernel merges the splits of each (b, g) and
// folds exp(sink) into the denominator exactly once.  When every sequence has
// a single split (a short window: 128 keys per sequence and kv head), the
// split kernel folds the sink itself and writes the output: one launch.
// The same kernel reads a paged cache through a block table (the producer maps
// each 64-key tile to its block's rows); kv_append_paged_kernel writes new
// tokens into such a cache.  Several new tokens of one sequence share a CTA:
// the M side holds (token, head) rows -- two tokens fill the 16 rows at G = 8,
// four fill two M fragments -- each row masking keys past its own position, so
// the cache is streamed once per CTA, not once per token.
#pragma once

#include "host_util.cuh"
#include "rope_qk.cuh"
#include "sm100_ptx.cuh"
#include "warp_mma.cuh"

namespace gptoss {

constexpr int kDecTileKeys = 64;       // keys per pipeline stage
constexpr int kDecConsumerWarps = 4;   // 16 keys of a stage each
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;
constexpr int kDecMaxGroup = 16;  // query heads per kv head
constexpr int kDecMaxRows = 32;   // query rows of a CTA: two 16-row M fragments

// Per head size kD (64 or 128): a stage holds one 64-key tile of K and one of
// V, each kD / 64 halves of 64 features (a 128B-swizzled 64-row TMA box,
// 8 KB); 96 KB of stages either way.
constexpr int kDecShortStages = 2;  // K / V ring of short key ranges (see DecodeSmem)

template <int kD>
struct DecCfg {
  static constexpr int kTileBytes = kDecTileKeys * kD * 2;
  static constexpr int kHalfBytes = kDecTileKeys * 64 * 2;
  static constexpr int kStages = kD == 64 ? 6 : 3;
};

struct DecodeParams {
  CUtensorMap tmap_k;  // dims (64, Hkv, Lmax, B), box (64, 1, 64, 1)
  CUtensorMap tmap_v;
  const __nv_bfloat16* q;  // [B, Hq, 64]
  __nv_bfloat16* out;      // [B, Hq, 64]
  float* lse;              // [B, Hq] nullable
  const int32_t* seqlens;  // [B]
  const float* sinks;      // [Hq]
  float* ws_o;             // [B, Hkv, nsplit, G, 64]
  float* ws_ml;            // [B, Hkv, nsplit, G, 2]
  int B, Lmax, Hq, Hkv, G, window, chunk, nsplit;
  int direct;  // one split per sequence: fold the sink and write out / lse here, no merge launch
  // query tokens per sequence: query token i of cache row b is the virtual
  // sequence b * q_len + i (q / out / lse row, workspace slot); it sees the
  // first len_b - (q_len - 1 - i) keys (causal among the new tokens).  One CTA
  // serves tpc consecutive tokens of a sequence (tpc * G query rows), so the
  // grid's z runs over B * n_slices, n_slices = ceil(q_len / tpc).
  int q_len, tpc, n_slices;
  // paged cache (block_table != nullptr): the K / V tensor maps cover the pools
  // [num_blocks * block_size, Hkv, 64]; token p of sequence b is row
  // block_table[b * max_blocks + p / block_size] * block_size + p % block_size
  const int32_t* block_table;
  int max_blocks, block_size, num_blocks;
  float scale_log2;
  uint64_t wait_ns;
  RopeTable tab;
};

// Split count and chunk length for a decode launch.  They depend only on the
// cache shape (not on the window), so the workspace sized for window 0 also
// covers every window.
__host__ __device__ inline int decode_chunk(int B, int Lmax, int Hkv) {
  // aim at about 16 CTAs per SM over the whole launch, chunks of 256..4096 keys
  const long long bh = static_cast<long long>(B) * Hkv;
  long long c = (static_cast<long long>(Lmax) * bh + 2367) / 2368;
  c = (c + kDecTileKeys - 1) / kDecTileKeys * kDecTileKeys;
  if (c < 256) c = 256;
  if (c > 4096) c = 4096;
  return static_cast<int>(c);
}

// kStages: the K / V ring; short key ranges (a 128-key window: at most three
// tiles) take a smaller ring, so more CTAs fit on an SM.
template <int kD, int kStages = DecCfg<kD>::kStages>
struct __align__(1024) DecodeSmem {
  uint8_t k[kStages][DecCfg<kD>::kTileBytes];
  uint8_t v[kStages][DecCfg<kD>::kTileBytes];  // directly after k (the merge uses both)
  __nv_bfloat16 q[kDecMaxRows][kD + 8];  // rotated query rows, padded
  float wm[kDecConsumerWarps][kDecMaxRows];
  float wl[kDecConsumerWarps][kDecMaxRows];
  uint64_t full[kStages];
  uint64_t empty[kStages];
};
// the four warps' partial outputs reuse the K and V stages at the end
template <int kD, int kStages>
constexpr bool dec_merge_fits = kDecConsumerWarps * kDecMaxRows * kD * 4 <= 2 * kStages * DecCfg<kD>::kTileBytes;

// The query tokens one CTA serves and the keys they see.  CTA z = (b, slice)
// takes new tokens tok0 .. tok0 + ntok - 1 of sequence b; its query rows are
// (token t, head h) -> row t * G + h.  Token t sees keys [lo_t, n_t) with
// n_t = n_first + t; the CTA streams the union [lo_first, n_last) split into
// chunks, and each row masks the keys outside its own range.
struct DecodeRows {
  int b, tok0, ntok, n_first, lo_first;
};

__device__ __forceinline__ DecodeRows decode_rows(const DecodeParams& p, int z) {
  DecodeRows r;
  r.b = z / p.n_slices;
  r.tok0 = (z - r.b * p.n_slices) * p.tpc;
  r.ntok = min(p.tpc, p.q_len - r.tok0);
  r.n_first = __ldg(p.seqlens + r.b) - (p.q_len - 1 - r.tok0);
  r.lo_first = p.window > 0 ? max(0, r.n_first - p.window) : 0;
  return r;
}

// RM = 16-row M fragments of query rows (1: up to 16 rows, 2: up to 32);
// kD = head size (64 or 128).
template <int RM, int kD, int kStages = DecCfg<kD>::kStages>
__global__ void __launch_bounds__(kDecThreads) attn_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  static_assert(dec_merge_fits<kD, kStages>, "the warps' partial outputs must fit in the K / V stages");
  constexpr int kHalf = DecCfg<kD>::kHalfBytes;
  constexpr int kPairsD = kD / 2;
  extern __shared__ uint8_t smem_raw[];
  DecodeSmem<kD, kStages>& sm = *reinterpret_cast<DecodeSmem<kD, kStages>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int g = blockIdx.x, split = blockIdx.y;
  const DecodeRows cr = decode_rows(p, blockIdx.z);
  // cache_seqlens[b]: the q_len new tokens fit in the cache, 1 <= len <= Lmax
  // (a failed check leaves this CTA's rows and partials unwritten)
  if (!index_ok(cr.n_first >= 1 && cr.n_first + p.q_len - 1 - cr.tok0 <= p.Lmax)) return;
  const int b = cr.b;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.G;
  const int n_last = cr.n_first + cr.ntok - 1;
  const int k_begin = cr.lo_first + split * p.chunk;
  const int k_end = min(n_last, k_begin + p.chunk);
  // paged: tiles start on 64-key boundaries (block_size is a multiple of 64,
  // so a tile never straddles two blocks); keys before k_begin are masked
  const int k_tile0 = p.block_table != nullptr ? (k_begin & ~(kDecTileKeys - 1)) : k_begin;
  if (k_begin >= k_end) {  // this split is past the sequence: the merge skips it
    if (p.direct) {        // (only an empty cache reaches here): the sink alone, O = 0
      for (int idx = threadIdx.x; idx < cr.ntok * G * kD; idx += kDecThreads) {
        const int row = idx / kD, t = row / G, head = g * G + row % G;
        const int64_t vb = static_cast<int64_t>(b) * p.q_len + cr.tok0 + t;
        p.out[(vb * p.Hq + head) * kD + idx % kD] = __float2bfloat16_rn(0.f);
        if (p.lse != nullptr && idx % kD == 0) p.lse[vb * p.Hq + head] = __ldg(p.sinks + head);
      }
    }
    return;
  }
  const int ntile = (k_end - k_tile0 + kDecTileKeys - 1) / kDecTileKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kDecConsumerWarps);
    }
    fence_mbar_init();
  }
  // rotated query rows of this CTA (zero rows past its tokens); token t's
  // query sits at position n_first + t - 1
  for (int idx = threadIdx.x; idx < 16 * RM * kPairsD; idx += kDecThreads) {
    const int row = idx / kPairsD, j = idx % kPairsD;
    const int t = row / G;
    float x = 0.f, y = 0.f;
    if (t < cr.ntok) {
      const int64_t vb = static_cast<int64_t>(b) * p.q_len + cr.tok0 + t;
      const __nv_bfloat16* qr = p.q + (vb * p.Hq + g * G + row % G) * kD;
      x = __bfloat162float(qr[rope_feature_a(j, p.tab.R)]);
      y = __bfloat162float(qr[rope_feature_b(j, p.tab.R)]);
      if (p.tab.enabled && j < p.tab.R) {
        const float2 cs = rope_cs(cr.n_first + t - 1, p.tab.inv_freq[j], p.tab.conc);
        const float xr = x * cs.x - y * cs.y;
        const float yr = y * cs.x + x * cs.y;
        x = xr;
        y = yr;
      }
    }
    sm.q[row][rope_feature_a(j, p.tab.R)] = __float2bfloat16_rn(x);
    sm.q[row][rope_feature_b(j, p.tab.R)] = __float2bfloat16_rn(y);
  }
  __syncthreads();

  if (warp == kDecConsumerWarps) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      tma_prefetch_desc(&p.tmap_k);
      tma_prefetch_desc(&p.tmap_v);
      for (int it = 0; it < ntile; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&sm.empty[s], ((it / kStages) & 1) ^ 1, p.wait_ns)) break;
        mbar_arrive_expect_tx(&sm.full[s], 2 * DecCfg<kD>::kTileBytes);
        const int key0 = k_tile0 + it * kDecTileKeys;
        int row = key0, bat = b;
        if (p.block_table != nullptr) {
          // a block index outside the pool (or a length past the table) reads
          // the tensor map's zero fill: the row coordinate is put past its end
          const int j = key0 / p.block_size;
          const int blk = j < p.max_blocks ? __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + j) : -1;
          row = (blk >= 0 && blk < p.num_blocks) ? blk * p.block_size + key0 % p.block_size
                                                  : p.num_blocks * p.block_size;
          bat = 0;
        }
#pragma unroll
        for (int hf = 0; hf < kD / 64; ++hf) {
          tma_load_4d(sm.k[s] + hf * kHalf, &p.tmap_k, &sm.full[s], 64 * hf, g, row, bat);
          tma_load_4d(sm.v[s] + hf * kHalf, &p.tmap_v, &sm.full[s], 64 * hf, g, row, bat);
        }
      }
      // drain: every issued stage must land before the CTA may exit
      const int first = ntile > kStages ? ntile - kStages : 0;
      for (int it = first; it < ntile; ++it)
        mbar_wait(&sm.full[it % kStages], (it / kStages) & 1, p.wait_ns);
    }
    return;
  }

  // ---------------- consumer warps ----------------
  const int gr = lane >> 2, tq = lane & 3;  // fragment row / column-pair index
  // query A fragments of M fragment mi: rows 16 mi + gr and 16 mi + gr + 8
  uint32_t qa[RM][kD / 16][4];
  // each of this thread's rows (mi, half) sees keys [klo, khi): its token's
  // range cut to this split; rows past the CTA's tokens see none
  int klo[RM][2], khi[RM][2];
#pragma unroll
  for (int mi = 0; mi < RM; ++mi) {
#pragma unroll
    for (int kt = 0; kt < kD / 16; ++kt) {
      const int c0 = kt * 16 + 2 * tq;
      qa[mi][kt][0] = *reinterpret_cast<const uint32_t*>(&sm.q[16 * mi + gr][c0]);
      qa[mi][kt][1] = *reinterpret_cast<const uint32_t*>(&sm.q[16 * mi + gr + 8][c0]);
      qa[mi][kt][2] = *reinterpret_cast<const uint32_t*>(&sm.q[16 * mi + gr][c0 + 8]);
      qa[mi][kt][3] = *reinterpret_cast<const uint32_t*>(&sm.q[16 * mi + gr + 8][c0 + 8]);
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int t = (16 * mi + gr + 8 * hf) / G;
      const int n_t = cr.n_first + t;
      const int lo_t = p.window > 0 ? max(0, n_t - p.window) : 0;
      klo[mi][hf] = max(k_begin, lo_t);
      khi[mi][hf] = t < cr.ntok ? min(k_end, n_t) : k_begin;
    }
  }
  float o[RM][kD / 8][4];
  float m[RM][2], l[RM][2];  // running max (log2 units) and this thread's share of the sums
#pragma unroll
  for (int mi = 0; mi < RM; ++mi) {
#pragma unroll
    for (int dt = 0; dt < kD / 8; ++dt) o[mi][dt][0] = o[mi][dt][1] = o[mi][dt][2] = o[mi][dt][3] = 0.f;
    m[mi][0] = m[mi][1] = -INFINITY;
    l[mi][0] = l[mi][1] = 0.f;
  }

  for (int it = 0; it < ntile; ++it) {
    const int s = it % kStages;
    if (!mbar_wait(&sm.full[s], (it / kStages) & 1, p.wait_ns)) break;
    const uint32_t kb = smem_u32(sm.k[s]);
    const uint32_t vb = smem_u32(sm.v[s]);
    const int r0 = warp * 16;  // first key row of this warp in the tile
    // S = Q K^T for two 8-key blocks; each K fragment serves every M fragment
    float sc[RM][2][4];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
      for (int mi = 0; mi < RM; ++mi) sc[mi][nb][0] = sc[mi][nb][1] = sc[mi][nb][2] = sc[mi][nb][3] = 0.f;
      const int row = r0 + nb * 8 + (lane & 7);
#pragma unroll
      for (int kp = 0; kp < kD / 32; ++kp) {  // 32 features per step; half kp / 2 of the row
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sw128_addr(kb + (kp >> 1) * kHalf, row, (kp & 1) * 4 + (lane >> 3)), b0, b1, b2, b3);
#pragma unroll
        for (int mi = 0; mi < RM; ++mi) {
          mma_bf16_16816(sc[mi][nb], qa[mi][2 * kp], b0, b1);
          mma_bf16_16816(sc[mi][nb], qa[mi][2 * kp + 1], b2, b3);
        }
      }
    }
    const int key_base = k_tile0 + it * kDecTileKeys + r0;
    float pr[RM][2][4];
#pragma unroll
    for (int mi = 0; mi < RM; ++mi) {
      // mask keys outside each row's range, scale into log2 units
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key_base + nb * 8 + 2 * tq + (e & 1);
          const int hf = e >> 1;
          sc[mi][nb][e] = (key >= klo[mi][hf] && key < khi[mi][hf]) ? sc[mi][nb][e] * p.scale_log2 : -INFINITY;
        }
      // online softmax, rows gr (e = 0, 1) and gr + 8 (e = 2, 3)
      float mx0 = fmaxf(fmaxf(sc[mi][0][0], sc[mi][0][1]), fmaxf(sc[mi][1][0], sc[mi][1][1]));
      float mx1 = fmaxf(fmaxf(sc[mi][0][2], sc[mi][0][3]), fmaxf(sc[mi][1][2], sc[mi][1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float n0 = fmaxf(m[mi][0], mx0), n1 = fmaxf(m[mi][1], mx1);
      const float b0s = n0 == -INFINITY ? 0.f : n0;  // safe subtrahends
      const float b1s = n1 == -INFINITY ? 0.f : n1;
      const float a0 = ex2_approx(m[mi][0] - b0s), a1 = ex2_approx(m[mi][1] - b1s);
      m[mi][0] = n0;
      m[mi][1] = n1;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        pr[mi][nb][0] = ex2_approx(sc[mi][nb][0] - b0s);
        pr[mi][nb][1] = ex2_approx(sc[mi][nb][1] - b0s);
        pr[mi][nb][2] = ex2_approx(sc[mi][nb][2] - b1s);
        pr[mi][nb][3] = ex2_approx(sc[mi][nb][3] - b1s);
      }
      l[mi][0] = l[mi][0] * a0 + (pr[mi][0][0] + pr[mi][0][1] + pr[mi][1][0] + pr[mi][1][1]);
      l[mi][1] = l[mi][1] * a1 + (pr[mi][0][2] + pr[mi][0][3] + pr[mi][1][2] + pr[mi][1][3]);
#pragma unroll
      for (int dt = 0; dt < kD / 8; ++dt) {
        o[mi][dt][0] *= a0;
        o[mi][dt][1] *= a0;
        o[mi][dt][2] *= a1;
        o[mi][dt][3] *= a1;
      }
    }
    // Rows of this warp past the sequence end get P = 0, but 0 x NaN is NaN:
    // those rows of a cache (a paged pool's unused rows above all) may hold
    // anything, so the warp zeroes its own V rows there before P V.
    const bool tail = key_base + 15 >= k_end;
    if (tail) {
      for (int idx = lane; idx < 16 * 8 * (kD / 64); idx += 32) {  // halves x 16 rows x 8 chunks of 16 bytes
        const int hf = idx >> 7, rr = (idx >> 3) & 15, ch = idx & 7;
        if (key_base + rr >= k_end)
          *reinterpret_cast<uint4*>(sm.v[s] + hf * kHalf + (r0 + rr) * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
    }
    // P as the A operand (16 query rows x 16 keys per M fragment)
    uint32_t pa[RM][4];
#pragma unroll
    for (int mi = 0; mi < RM; ++mi) {
      pa[mi][0] = pack_bf16(pr[mi][0][0], pr[mi][0][1]);
      pa[mi][1] = pack_bf16(pr[mi][0][2], pr[mi][0][3]);
      pa[mi][2] = pack_bf16(pr[mi][1][0], pr[mi][1][1]);
      pa[mi][3] = pack_bf16(pr[mi][1][2], pr[mi][1][3]);
    }
    // O += P V over 8 feature blocks of 8; each V fragment serves every M fragment
#pragma unroll
    for (int dp = 0; dp < kD / 16; ++dp) {  // 16 features per step; half dp / 4 of the row
      uint32_t v0, v1, v2, v3;
      const int row = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
      ldsm_x4_t(sw128_addr(vb + (dp >> 2) * kHalf, row, 2 * (dp & 3) + (lane >> 4)), v0, v1, v2, v3);
#pragma unroll
      for (int mi = 0; mi < RM; ++mi) {
        mma_bf16_16816(o[mi][2 * dp], pa[mi], v0, v1);
        mma_bf16_16816(o[mi][2 * dp + 1], pa[mi], v2, v3);
      }
    }
    if (tail) fence_proxy_async_smem();  // the zeroed rows before the next TMA write of the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[s]);
  }

  // ---------------- merge the four warps ----------------
  // The per-warp accumulators reuse the K and V stages once every warp is
  // done (4 warps x 32 rows x kD floats: at most 64 KB of the 96 KB).
  named_barrier_sync(1, kDecConsumerWarps * 32);
  float(*wo)[kDecMaxRows][kD] = reinterpret_cast<float(*)[kDecMaxRows][kD]>(&sm.k[0][0]);
#pragma unroll
  for (int mi = 0; mi < RM; ++mi) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float lv = l[mi][hf];
      lv += __shfl_xor_sync(0xffffffffu, lv, 1);
      lv += __shfl_xor_sync(0xffffffffu, lv, 2);
      if (tq == 0) {
        sm.wm[warp][16 * mi + gr + 8 * hf] = m[mi][hf];
        sm.wl[warp][16 * mi + gr + 8 * hf] = lv;
      }
    }
#pragma unroll
    for (int dt = 0; dt < kD / 8; ++dt) {
      wo[warp][16 * mi + gr][dt * 8 + 2 * tq] = o[mi][dt][0];
      wo[warp][16 * mi + gr][dt * 8 + 2 * tq + 1] = o[mi][dt][1];
      wo[warp][16 * mi + gr + 8][dt * 8 + 2 * tq] = o[mi][dt][2];
      wo[warp][16 * mi + gr + 8][dt * 8 + 2 * tq + 1] = o[mi][dt][3];
    }
  }
  named_barrier_sync(1, kDecConsumerWarps * 32);
  const int tid = threadIdx.x;  // 128 consumer threads: (row, 4 features)
  for (int idx = tid; idx < 16 * RM * (kD / 4); idx += kDecConsumerWarps * 32) {
    const int row = idx / (kD / 4), d4 = (idx % (kD / 4)) * 4;
    const int t = row / G, h = row - t * G;
    if (t >= cr.ntok) continue;
    const int64_t vbq = static_cast<int64_t>(b) * p.q_len + cr.tok0 + t;  // virtual sequence of the row
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, sm.wm[w][row]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) {
      const float sc = ex2_approx(sm.wm[w][row] - Ms);
      L += sm.wl[w][row] * sc;
      acc.x += wo[w][row][d4] * sc;
      acc.y += wo[w][row][d4 + 1] * sc;
      acc.z += wo[w][row][d4 + 2] * sc;
      acc.w += wo[w][row][d4 + 3] * sc;
    }
    if (p.direct) {
      // the only split of this (b, g): fold exp(sink) here as the merge would
      const int head = g * G + h;
      const float sink = __ldg(p.sinks + head) * kLog2e;
      const float Mt = fmaxf(M, sink);
      const float Mts = Mt == -INFINITY ? 0.f : Mt;
      const float sc = M == -INFINITY ? 0.f : ex2_approx(M - Mts);
      const float Lt = L * sc + ex2_approx(sink - Mts);
      const float inv = sc / Lt;
      uint2 r;
      r.x = pack_bf16(acc.x * inv, acc.y * inv);
      r.y = pack_bf16(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(p.out + (vbq * p.Hq + head) * kD + d4) = r;
      if (p.lse != nullptr && d4 == 0) p.lse[vbq * p.Hq + head] = (Mt + log2f(Lt)) * kLn2;
      continue;
    }
    const int64_t slot = ((vbq * p.Hkv + g) * p.nsplit + split) * G + h;
    *reinterpret_cast<float4*>(p.ws_o + slot * kD + d4) = acc;
    if (d4 == 0) {
      p.ws_ml[slot * 2] = M;
      p.ws_ml[slot * 2 + 1] = L;
    }
  }
}

// Merge the splits of one (virtual sequence, g): fold exp(sink) once,
// normalise, write bf16.  The splits are those of the sequence's CTA group:
// chunks of the union of its tokens' key ranges.
template <int kD>
__global__ void __launch_bounds__(256) attn_decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  const int g = blockIdx.x, vb = blockIdx.y;  // virtual sequence (cache row, query token)
  const int b = vb / p.q_len, tok = vb - b * p.q_len;
  const DecodeRows cr = decode_rows(p, b * p.n_slices + tok / p.tpc);
  if (!index_ok(cr.n_first >= 1 && cr.n_first + p.q_len - 1 - cr.tok0 <= p.Lmax)) return;
  const int n_last = cr.n_first + cr.ntok - 1;
  const int nsp = min(p.nsplit, (n_last - cr.lo_first + p.chunk - 1) / p.chunk);
  const int G = p.G;
  for (int idx = threadIdx.x; idx < G * (kD / 2); idx += 256) {
    const int h = idx / (kD / 2), d2 = (idx % (kD / 2)) * 2;
    const int head = g * G + h;
    const float sink = __ldg(p.sinks + head) * kLog2e;
    const int64_t base = (static_cast<int64_t>(vb) * p.Hkv + g) * p.nsplit;
    float M = sink;
    for (int s = 0; s < nsp; ++s) M = fmaxf(M, p.ws_ml[((base + s) * G + h) * 2]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float L = ex2_approx(sink - Ms);
    float ox = 0.f, oy = 0.f;
    for (int s = 0; s < nsp; ++s) {
      const int64_t slot = (base + s) * G + h;
      const float sc = ex2_approx(p.ws_ml[slot * 2] - Ms);
      L += p.ws_ml[slot * 2 + 1] * sc;
      const float2 ov = *reinterpret_cast<const float2*>(p.ws_o + slot * kD + d2);
      ox += ov.x * sc;
      oy += ov.y * sc;
    }
    const float inv = 1.f / L;
    __nv_bfloat162 r;
    r.x = __float2bfloat16_rn(ox * inv);
    r.y = __float2bfloat16_rn(oy * inv);
    *reinterpret_cast<__nv_bfloat162*>(p.out + (static_cast<int64_t>(vb) * p.Hq + head) * kD + d2) = r;
    if (p.lse != nullptr && d2 == 0) p.lse[static_cast<int64_t>(vb) * p.Hq + head] = (M + log2f(L)) * kLn2;
  }
}

// KV-cache append: sequence b's q_len new tokens (positions cache_seqlens[b]
// - q_len .. cache_seqlens[b] - 1) into a paged cache -- the keys rotated
// (the cache holds post-RoPE keys, bf16), the values as given.  Block (b, i):
// new token i of sequence b; thread (g, j): pair j of kv head g.
struct AppendParams {
  const __nv_bfloat16* k_new;  // [B, q_len, Hkv, D]
  const __nv_bfloat16* v_new;
  const int32_t* seqlens;      // [B]
  const int32_t* block_table;  // [B, max_blocks]
  __nv_bfloat16* k_pool;       // [num_blocks * block_size, Hkv, D]
  __nv_bfloat16* v_pool;
  int B, q_len, Hkv, D, max_blocks, block_size, num_blocks;
  RopeTable tab;
};


__global__ void kv_append_paged_kernel(const __grid_constant__ AppendParams p) {
  const int b = blockIdx.x, tok = blockIdx.y;
  const int g = threadIdx.x / (p.D / 2), j = threadIdx.x % (p.D / 2);
  const int pos = __ldg(p.seqlens + b) - p.q_len + tok;
  const int jb = pos >= 0 ? pos / p.block_size : -1;
  const int blk = (jb >= 0 && jb < p.max_blocks) ? __ldg(p.block_table + static_cast<int64_t>(b) * p.max_blocks + jb) : -1;
  if (blk < 0 || blk >= p.num_blocks) {  // nothing is written outside the pool
    if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusBadIndex);
    return;
  }
  const int64_t off = (static_cast<int64_t>(blk) * p.block_size + pos % p.block_size) * p.Hkv * p.D +
                      static_cast<int64_t>(g) * p.D;
  const int64_t src = ((static_cast<int64_t>(b) * p.q_len + tok) * p.Hkv + g) * p.D;
  const int fa = rope_feature_a(j, p.tab.R), fb = rope_feature_b(j, p.tab.R);
  float x = __bfloat162float(p.k_new[src + fa]), y = __bfloat162float(p.k_new[src + fb]);
  if (p.tab.enabled && j < p.tab.R) {
    const float2 cs = rope_cs(pos, p.tab.inv_freq[j], p.tab.conc);
    const float xr = x * cs.x - y * cs.y, yr = y * cs.x + x * cs.y;
    x = xr;
    y = yr;
  }
  p.k_pool[off + fa] = __float2bfloat16_rn(x);
  p.k_pool[off + fb] = __float2bfloat16_rn(y);
  p.v_pool[off + fa] = p.v_new[src + fa];
  p.v_pool[off + fb] = p.v_new[src + fb];
}

}  // namespace gptoss
