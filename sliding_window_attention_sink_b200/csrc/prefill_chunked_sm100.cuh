// prefill_chunked_sm100.cuh -- global-attention (and wide-window) prefill as a
// persistent, warp-specialised pipeline on sm_100a.
//
// Operation: "MiMo-V2-Flash Technical Report" summary (mlpod.com), section
// 2.2.2 (a sink term in the softmax denominator, a max term for stability)
// over the global-attention layers of section 2.2 (every earlier key of the
// sequence is visible), and over sliding windows too wide for the ring kernel.
//
// Work: one 128-row tile = TM tokens x G query heads of one kv head (GQA
// packing, as in the sliding-window kernel). A tile's keys [lo, last token]
// stream through shared memory in chunks of 128 keys; for each chunk the
// S = Q K^T and O += P V contractions run on tcgen05 with O accumulating in
// TMEM across the chunks. Tiles are dealt to the persistent CTAs round-robin
// in order of decreasing work (the last token tiles of a sequence are the
// heaviest under the causal mask).
//
// Online softmax with a lazy rescale: P = exp2(x - m_used) with a per-row
// reference max m_used that only moves when a chunk's max exceeds it by more
// than kRescaleLog2 (log2 units; P then stays below 2^8, well inside bf16 and
// fp32). When it moves, the warp waits for the previous PV MMA and rescales its
// columns of O (and its row sums) by exp2(m_old - m_new) in TMEM. The final
// O / l and LSE = m_used + log2(l) are exact whatever m_used is.
//
//   warps 0-7   two softmax warpgroups. Each thread owns one row (TMEM lane);
//               group hw loads only columns [64 hw, 64 hw + 64) of the chunk,
//               takes the row's chunk max from the max warps, exponentiates
//               its columns and writes its half of P.
//   warps 8-11  max and epilogue: per chunk, the masked row max over all 128
//               columns, handed to the softmax groups through shared memory
//               (two slots, one chunk ahead where S allows); after a tile's
//               last PV, O / l -> bf16 -> global (one row per thread) and the
//               LSE. The exponentials (16 per clock per SM: a chunk's 16384
//               take as long as its MMAs) then run while the next chunk's
//               maximum is found, instead of after it.
//   warp 12     TMA producer: Q tile (2 stages), K and V chunks (2 stages
//               each; K of chunk n goes out before V of chunk n - 1).
//   warp 13     TMEM allocation; S = Q K^T into S buffer (chunk & 1).
//   warp 14     O += P V (P from its own TMEM buffer, V MN-major).
//
// TMEM columns: S buffers [0, 128) and [128, 256), O [256, 256 + D), P buffers
// [384, 448) and [448, 512) (bf16 pairs, 8 columns per 16 keys).
//
// Every wait is bounded (see mbar_wait); nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

// Pipeline timeline hooks: compiled out unless SWA_CHUNK_TRACE is defined (a
// profiling build then supplies swa_chunk_trace: clock64 stamps of CTA 0,
// [role][chunk][event], roles 0 producer, 1 S issuer, 2 PV issuer, 3 and 4 the
// softmax groups, 5 epilogue; and swa_chunk_cta: globaltimer at each CTA's
// start and end).
#ifdef SWA_CHUNK_TRACE
__device__ unsigned long long* swa_chunk_trace;
__device__ unsigned long long* swa_chunk_cta;
#define CHUNK_TRACE(role, j, ev)                                                          \
  do {                                                                                    \
    if (blockIdx.x == 0 && (j) < 256)                                                     \
      swa_chunk_trace[((role) * 256 + (j)) * 8 + (ev)] =                                  \
          static_cast<unsigned long long>(clock64());                                     \
  } while (0)
#define CHUNK_CTA(ev)                                                                     \
  do {                                                                                    \
    if (threadIdx.x == 0) swa_chunk_cta[blockIdx.x * 2 + (ev)] = globaltimer_ns();        \
  } while (0)
#else
#define CHUNK_TRACE(role, j, ev) \
  do {                           \
    (void)(role);                \
  } while (0)
#define CHUNK_CTA(ev) \
  do {                \
  } while (0)
#endif

constexpr int kChunkThreads = 480;   // 15 warps
constexpr int kChunkKeys = 128;      // keys per chunk (N of S, K of PV)
constexpr float kRescaleLog2 = 8.f;  // lazy-rescale threshold (log2 units)

struct ChunkParams {
  const int32_t* cu_seqlens;
  int num_seqs;
  int total;
  int Hq, Hkv, G, TM;
  int window;         // <= 0: full causal prefix; > 0: sliding window
  int n_tok_tiles;
  int n_tiles;        // n_tok_tiles * Hkv
  const float* sink;
  float scale_log2;
  __nv_bfloat16* o;   // [total, Hq, D]
  float* lse;         // [Hq, total] or null
  uint32_t q_box_bytes;  // bytes of one 64-column Q box
};

// Dynamic smem bytes (1 KB alignment slack): two stages each of Q, K and V.
__host__ __device__ inline size_t chunked_smem_bytes(int D) {
  return 1024 + 3 * 2 * static_cast<size_t>(D / 64) * 16384;
}

template <int D>
__global__ void __launch_bounds__(kChunkThreads, 1)
    prefill_chunked_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const ChunkParams p) {
  constexpr int NCH = D / 64;
  constexpr uint32_t CH = 16384;               // one 64-dim chunk: 128 rows x 128 bytes
  constexpr int HALF = kChunkKeys / 2;         // columns per softmax warpgroup
  constexpr uint32_t o_col = 2 * kChunkKeys;   // after the two S buffers
  constexpr uint32_t p_col = 384;              // two P buffers of 64 columns
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full[2], q_empty[2], k_full[2], k_empty[2];
  __shared__ __align__(8) uint64_t v_full[2], v_empty[2];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2];
  __shared__ __align__(8) uint64_t o_full, o_empty, l_full, l_free;
  __shared__ float red_lr[2][128], red_lx[2][128], m_s[128];
  // row max of chunk n (raw S units, masked) in slot n & 1, from the max warps
  __shared__ float m_chunk[2][128];
  __shared__ __align__(8) uint64_t mx_full[2], mx_empty[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &abort_sh;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base;               // [stage][NCH] x CH
  const uint32_t sK = sQ + 2 * NCH * CH;
  const uint32_t sV = sK + 2 * NCH * CH;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&q_empty[s]), 1);
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_empty[s]), 12);  // 8 softmax warps + 4 max warps
      mbar_init(smem_u32(&p_full[s]), 8);
      mbar_init(smem_u32(&p_empty[s]), 1);
      mbar_init(smem_u32(&mx_full[s]), 4);
      mbar_init(smem_u32(&mx_empty[s]), 8);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), 4);
    mbar_init(smem_u32(&l_full), 8);
    mbar_init(smem_u32(&l_free), 4);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  CHUNK_CTA(0);

  // the k-th tile of this CTA: heaviest (last) token tiles first
  auto tile_of = [&](int k, int& g, int& tb) {
    const int f = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    const int rank = f / p.Hkv;
    g = f - rank * p.Hkv;
    tb = p.n_tok_tiles - 1 - rank;
  };
  const int ntile = (p.n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                    static_cast<int>(gridDim.x);
  // keys of a tile: [lo, last token] in chunks of 128 (the first visible key
  // never decreases along the packed token axis)
  auto tile_keys = [&](int tb, int& lo, int& nchunk) {
    const int t0 = tb * p.TM;
    const int t_last = min(t0 + p.TM, p.total) - 1;
    lo = first_key(p.cu_seqlens, p.num_seqs, p.window, t0);
    nchunk = (t_last - lo + kChunkKeys) / kChunkKeys;
  };

  if (warp < 8) {
    // ===================== softmax (two warpgroups) ==========================
    const int hw = warp >> 2;              // which 64 columns this group exponentiates
    const int r = 32 * (warp & 3) + lane;  // TMEM lane == tile row
    const int tok = r / p.G, hh = r - tok * p.G;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    int n = 0;  // chunk counter over the CTA's tiles; buffers n & 1
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const int t0 = tb * p.TM;
      const int i = t0 + tok;
      const int h = g * p.G + hh;
      const bool valid = i < p.total;
      int row_lo = 0, row_hi = -1;  // rows past the end see no key
      if (valid) {
        row_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, i);
        row_hi = i;
      }
      const int t_last = min(t0 + p.TM, p.total) - 1;
      // keys visible to every row of the tile
      const int all_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, t_last);
      const int all_hi = t0;
      const float sink2 = (valid && p.sink != nullptr) ? __ldg(p.sink + h) * kLog2e : -INFINITY;
      float m_used = sink2;        // reference max of P (log2 units)
      float l_r = 0.f, l_x = 0.f;  // this group's sums relative to m_used
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1;
        const int trole = 3 + hw;
        const bool tr = (tid & 127) == 0;
        if (tr) CHUNK_TRACE(trole, n, 0);
        // the row's chunk max from the max warps
        if (!mbar_wait(smem_u32(&mx_full[b]), (n >> 1) & 1, abort) ||
            !mbar_wait(smem_u32(&s_full[b]), (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        const float cm_raw = m_chunk[b][r];
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&mx_empty[b]));
        tc_fence_after();
        if (tr) CHUNK_TRACE(trole, n, 1);
        const uint32_t tS = tmem + lane_off + b * kChunkKeys;
        // this group's columns of S
        uint32_t v[HALF];
        {
          const int cb = lo + c * kChunkKeys + hw * HALF;  // key of column 0 of this half
#pragma unroll
          for (int q = 0; q < HALF / 16; ++q) tmem_ld16_at(tS + hw * HALF + q * 16, &v[q * 16]);
          tmem_ld_wait();
          if (!(cb >= all_lo && cb + HALF - 1 <= all_hi)) {  // a row's edge is in this half
            const int cmin = row_lo - cb;
            const int cmax = row_hi - cb;
#pragma unroll
            for (int e = 0; e < HALF; ++e)
              if (e < cmin || e > cmax) v[e] = 0xff800000u;  // -inf
          }
        }
        // S of this chunk is in registers: the buffer may take S of chunk n + 2
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s_empty[b]));
        if (tr) CHUNK_TRACE(trole, n, 2);
        const float cm = cm_raw * p.scale_log2;
        // lazy rescale: the reference moves only when the max outgrows it
        const bool grow = cm > m_used + kRescaleLog2;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = grow ? cm : m_used;
          const float alpha = grow ? ex2(m_used - m_new) : 1.f;  // exp2(-inf) = 0
          // O holds the PVs of chunks before n once PV(n - 1) has completed
          // (PV(n - 3) has, since this group wrote P(n - 1) after it)
          if (c > 0 &&
              mbar_wait(smem_u32(&p_empty[(n - 1) & 1]), ((n - 1) >> 1) & 1, abort)) {
            __syncwarp();
            tc_fence_after();
            const uint32_t tO = tmem + lane_off + o_col + hw * (D / 2);
#pragma unroll
            for (int q = 0; q < D / 2; q += 16) {
              uint32_t w[16];
              tmem_ld16_at(tO + q, w);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
              tmem_st16(tO + q, w);
            }
          }
          l_r *= alpha;
          l_x *= alpha;
          m_used = m_new;
        }
        const float mb = (m_used == -INFINITY) ? 0.f : m_used;
        if (tr) CHUNK_TRACE(trole, n, 3);
        // P buffer b is free once PV(n - 2) has completed
        if (!mbar_wait(smem_u32(&p_empty[b]), ((n >> 1) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        if (tr) CHUNK_TRACE(trole, n, 4);
        // P = exp2(x - m_used) as bf16 pairs: this group's 32 columns
        uint64_t lr2 = 0, lx2 = 0;
        const uint64_t nm2 = f2_pack(-mb, -mb);
        const uint32_t tP = tmem + lane_off + p_col + b * HALF + hw * (HALF / 2);
#pragma unroll
        for (int q = 0; q < HALF; q += 16) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float t0f, t1f;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(v[q + e]), __uint_as_float(v[q + e + 1])),
                             sc2, nm2),
                      t0f, t1f);
            const float x0 = ex2(t0f), x1 = ex2(t1f);
            w[e >> 1] = pack_bf16x2(x0, x1);
            lr2 = f2_add(lr2, f2_pack(bf16lo_to_f32(w[e >> 1]), bf16hi_to_f32(w[e >> 1])));
            lx2 = f2_add(lx2, f2_pack(x0, x1));
          }
          tmem_st8(tP + q / 2, w);
        }
        {
          float a0, a1;
          f2_unpack(lr2, a0, a1);
          l_r += a0 + a1;
          f2_unpack(lx2, a0, a1);
          l_x += a0 + a1;
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[b]));
        if (tr) CHUNK_TRACE(trole, n, 5);
      }
      if (!ok) break;
      // tile done: this group's sums (group 0 adds the sink term) and the
      // reference max go to the epilogue once it has read the previous tile's
      const float mb = (m_used == -INFINITY) ? 0.f : m_used;
      if (hw == 0 && sink2 != -INFINITY) {
        const float ts = ex2(sink2 - mb);
        l_r += ts;
        l_x += ts;
      }
      if (!mbar_wait(smem_u32(&l_free), (k & 1) ^ 1, abort)) break;
      red_lr[hw][r] = l_r;
      red_lx[hw][r] = l_x;
      if (hw == 0) m_s[r] = mb;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_full));
    }
  } else if (warp < 12) {
    // =============== chunk maxima and epilogue (warps 8..11) ==================
    const int r = 32 * (warp & 3) + lane;
    const int tok = r / p.G, hh = r - tok * p.G;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tO = tmem + lane_off + o_col;
    // tile k's epilogue: O / l -> bf16 -> global, and the LSE
    auto drain = [&](int k) -> bool {
      int g, tb;
      tile_of(k, g, tb);
      if (tid == 256) CHUNK_TRACE(5, k, 0);
      if (!mbar_wait(smem_u32(&o_full), k & 1, abort)) return false;
      if (tid == 256) CHUNK_TRACE(5, k, 1);
      if (!mbar_wait(smem_u32(&l_full), k & 1, abort)) return false;
      if (tid == 256) CHUNK_TRACE(5, k, 2);
      __syncwarp();
      tc_fence_after();
      const float l = red_lr[0][r] + red_lr[1][r];
      const float lse2 = m_s[r] + lg2(red_lx[0][r] + red_lx[1][r]);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_free));
      const int i = tb * p.TM + tok;
      const int h = g * p.G + hh;
      const bool valid = i < p.total;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<size_t>(valid ? i : 0) * p.Hq + h) * D;
#pragma unroll
      for (int q = 0; q < D; q += 32) {
        uint32_t v[32];
        tmem_ld16_at(tO + q, &v[0]);
        tmem_ld16_at(tO + q + 16, &v[16]);
        tmem_ld_wait();
        if (q + 32 == D) {  // O is read: the next tile's PV may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&o_empty));
        }
        if (valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float* f = reinterpret_cast<const float*>(&v[u * 8]);
            uint4 w;
            w.x = pack_bf16x2(f[0] * inv_l, f[1] * inv_l);
            w.y = pack_bf16x2(f[2] * inv_l, f[3] * inv_l);
            w.z = pack_bf16x2(f[4] * inv_l, f[5] * inv_l);
            w.w = pack_bf16x2(f[6] * inv_l, f[7] * inv_l);
            *reinterpret_cast<uint4*>(orow + q + u * 8) = w;
          }
        }
      }
      if (valid && p.lse != nullptr) p.lse[static_cast<size_t>(h) * p.total + i] = lse2 * kLn2;
      if (tid == 256) CHUNK_TRACE(5, k, 3);
      return true;
    };
    int n = 0;  // chunk counter over the CTA's tiles, as the softmax counts
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const int t0 = tb * p.TM;
      const int i = t0 + tok;
      int row_lo = 0, row_hi = -1;  // rows past the end see no key
      if (i < p.total) {
        row_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, i);
        row_hi = i;
      }
      const int t_last = min(t0 + p.TM, p.total) - 1;
      // keys visible to every row of the tile
      const int all_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, t_last);
      const int all_hi = t0;
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1;
        if (!mbar_wait(smem_u32(&s_full[b]), (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + b * kChunkKeys;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          uint32_t v[HALF];
          const int cb = lo + c * kChunkKeys + hs * HALF;  // key of column 0 of this half
#pragma unroll
          for (int q = 0; q < HALF / 16; ++q) tmem_ld16_at(tS + hs * HALF + q * 16, &v[q * 16]);
          tmem_ld_wait();
          if (!(cb >= all_lo && cb + HALF - 1 <= all_hi)) {  // a row's edge is in this half
            const int cmin = row_lo - cb;
            const int cmax = row_hi - cb;
#pragma unroll
            for (int e = 0; e < HALF; ++e)
              if (e < cmin || e > cmax) v[e] = 0xff800000u;  // -inf
          }
#pragma unroll
          for (int e = 0; e < HALF; e += 4) {
            mx0 = max3(mx0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            mx1 = max3(mx1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s_empty[b]));
        // hand the max over once the softmax has read slot b's previous one
        if (!mbar_wait(smem_u32(&mx_empty[b]), ((n >> 1) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        m_chunk[b][r] = fmaxf(mx0, mx1);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&mx_full[b]));
        // the previous tile's epilogue, once this tile's first max is out
        // (the softmax needs it before it can finish the tile whose PV the
        // epilogue waits for)
        if (c == 0 && k > 0 && !drain(k - 1)) {
          ok = false;
          break;
        }
      }
    }
    if (ok && ntile > 0) drain(ntile - 1);
  } else if (warp == 12) {
    // ======================= TMA producer ====================================
    // Order: Q of a tile before its first K; K of chunk n before V of chunk
    // n - 1, so S can run ahead of PV.
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int n = 0;
      int pend_key = -1, pend_g = 0;  // V still to load for chunk n - 1
      auto load_v = [&](int m, int key0, int g) -> bool {
        const int st = m & 1;
        if (!mbar_wait(smem_u32(&v_empty[st]), ((m >> 1) & 1) ^ 1, abort)) return false;
        const uint32_t bar = smem_u32(&v_full[st]);
        mbar_arrive_expect_tx(bar, NCH * CH);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_load_3d(sV + (st * NCH + ch) * CH, &tm_v, bar, ch * 64, g, key0);
        return true;
      };
      bool ok = true;
      for (int k = 0; k < ntile && ok; ++k) {
        int g, tb, lo, nchunk;
        tile_of(k, g, tb);
        tile_keys(tb, lo, nchunk);
        const int qs = k & 1;
        if (!mbar_wait(smem_u32(&q_empty[qs]), ((k >> 1) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(smem_u32(&q_full[qs]), NCH * p.q_box_bytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_load_3d(sQ + (qs * NCH + ch) * CH, &tm_q, smem_u32(&q_full[qs]), ch * 64, g * p.G,
                      tb * p.TM);
        for (int c = 0; c < nchunk; ++c, ++n) {
          const int st = n & 1;
          const int key0 = lo + c * kChunkKeys;
          CHUNK_TRACE(0, n, 0);
          if (!mbar_wait(smem_u32(&k_empty[st]), ((n >> 1) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          const uint32_t bar = smem_u32(&k_full[st]);
          mbar_arrive_expect_tx(bar, NCH * CH);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_3d(sK + (st * NCH + ch) * CH, &tm_k, bar, ch * 64, g, key0);
          CHUNK_TRACE(0, n, 1);
          if (pend_key >= 0 && !load_v(n - 1, pend_key, pend_g)) {
            ok = false;
            break;
          }
          CHUNK_TRACE(0, n, 2);
          pend_key = key0;
          pend_g = g;
        }
      }
      if (ok && pend_key >= 0) load_v(n - 1, pend_key, pend_g);
    }
  } else if (warp == 13) {
    // ======================= S = Q K^T issuer ================================
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);
    const uint32_t idesc = idesc_bf16_f32(128, kChunkKeys, false, false);
    int n = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const int qs = k & 1;
      if (!mbar_wait(smem_u32(&q_full[qs]), (k >> 1) & 1, abort)) break;
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1;
        if (lane == 0) CHUNK_TRACE(1, n, 0);
        if (!mbar_wait(smem_u32(&s_empty[b]), ((n >> 1) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        if (lane == 0) CHUNK_TRACE(1, n, 1);
        if (!mbar_wait(smem_u32(&k_full[b]), (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t aq = kmaj | ((sQ + qs * NCH * CH) >> 4);
        const uint64_t bk = kmaj | ((sK + b * NCH * CH) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * CH + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tmem + b * kChunkKeys, aq + off, bk + off, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&s_full[b]));
          mma_commit(smem_u32(&k_empty[b]));
          if (c == nchunk - 1) mma_commit(smem_u32(&q_empty[qs]));
        }
        if (lane == 0) CHUNK_TRACE(1, n, 2);
        __syncwarp();
      }
    }
  } else if (warp == 14) {
    // ======================= O += P V issuer =================================
    const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
    // V as the MN-major B operand: 64-dim blocks CH apart (LBO), 8-key groups
    // 1024 bytes apart (SBO)
    const uint64_t mnmaj = smem_desc_sw128(0, CH, 1024);
    int n = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1;
        if (lane == 0) CHUNK_TRACE(2, n, 0);
        if (!mbar_wait(smem_u32(&p_full[b]), (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        if (lane == 0) CHUNK_TRACE(2, n, 1);
        if ((c == 0 && !mbar_wait(smem_u32(&o_empty), (k & 1) ^ 1, abort)) ||
            !mbar_wait(smem_u32(&v_full[b]), (n >> 1) & 1, abort)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t vd = mnmaj | ((sV + b * NCH * CH) >> 4);
        const uint32_t aP = tmem + p_col + b * HALF;  // P: 8 columns per 16 keys
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kChunkKeys / 16; ++kk)
            mma_bf16_ts(tmem + o_col, aP + kk * 8, vd + ((kk * 16 * 128) >> 4), idesc_pv,
                        (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&p_empty[b]));
          mma_commit(smem_u32(&v_empty[b]));
          if (c == nchunk - 1) mma_commit(smem_u32(&o_full));
        }
        if (lane == 0) CHUNK_TRACE(2, n, 2);
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  CHUNK_CTA(1);
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
