// prefill_sm100.cuh -- varlen prefill: causal GQA attention over a sliding
// window (or the full causal prefix) with a per-head sink logit, sm_100a.
//
// Operation: "MiMo-V2-Flash Technical Report" summary (mlpod.com), section
// 2.2.2 "Learnable Attention Sink Bias" (sink term in the softmax
// denominator, a max term for stability) and section 2.2.1 (window of 128).
// Per query row: m = max(s_h, max_j a_j), den = exp(s_h-m) + sum_j exp(a_j-m),
// o = sum_j exp(a_j-m)/den * v_j, lse = m + ln(den); a_j = scale * q.k_j.
//
// Tiling (B200-specific; the pages give no kernel):
// * GQA packing: one 128-row MMA tile = TM consecutive tokens x G query heads
//   of ONE kv head (TM = 128 / G). Row r <-> (token t0 + r / G, head g*G +
//   r % G). The Q tile is one 3-D TMA box [64 dims, G heads, TM tokens]. A
//   K/V tile is read once for all G heads of its group.
// * Key chunks of BN keys, BN a multiple of 16 (<= 256). For a sliding window
//   with W + TM - 1 <= 256, one chunk of BN = roundup16(W + TM - 1) covers
//   every key the tile needs (144 for W = 128, G = 8), so the MMA does 144/128
//   of the useful work instead of the 2x of a 128x128 query/key tiling.
//   Global layers loop over chunks of 128 keys.
// * S = Q K^T and O += P V on the 5th-generation tensor cores
//   (tcgen05.mma, bf16 in, f32 accumulate in TMEM). Operands are staged in
//   shared memory with the 128-byte swizzle: Q and K by TMA (K-major), V by
//   TMA and read MN-major by the PV MMA, P written by the softmax threads.
// * Softmax: thread r owns TMEM lane r (its row), so row max and row sum need
//   no shuffles. The running max starts at the sink logit and the running sum
//   at exp(0) = 1 for the sink term; when the max grows, O (in TMEM) and the
//   sum are rescaled.
// * Rows and keys are handled on the packed token axis: a tile may straddle a
//   sequence boundary; every row masks keys outside [its window start, itself]
//   and before its own sequence start.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx_sm100.cuh"

namespace swa {

struct PrefillParams {
  const int32_t* cu_seqlens;  // [num_seqs + 1]
  int num_seqs;
  int total;        // packed tokens
  int Hq, Hkv, G;   // G = Hq / Hkv
  int TM;           // tokens per tile (TM * G <= 128)
  int window;       // > 0 sliding window incl. self, <= 0 full causal
  int BN;           // keys per chunk (multiple of 16, 16..256)
  int n_tok_tiles;  // ceil(total / TM)
  int reverse;      // 1: process token tiles last-to-first (global layers)
  const float* sink;  // [Hq] or null
  float scale_log2;   // softmax_scale * log2(e)
  __nv_bfloat16* o;   // [total, Hq, D]
  float* lse;         // [Hq, total] or null
  uint32_t q_box_bytes;  // bytes one 64-column Q box writes (128 * TM * G)
  uint32_t tmem_cols;    // power of two >= o_col + D
  uint32_t o_col;        // TMEM column of the O accumulator
};

// The sequence containing packed token t: largest s with cu[s] <= t.
__device__ __forceinline__ int seq_of_token(const int32_t* cu, int num_seqs, int t) {
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// First key visible to token t: its own sequence start, or t - W + 1.
__device__ __forceinline__ int first_key(const int32_t* cu, int num_seqs, int window, int t) {
  const int s = seq_of_token(cu, num_seqs, t);
  int lo = __ldg(cu + s);
  if (window > 0) lo = max(lo, t - window + 1);
  return lo;
}

// first_key with the bounds [s_lo, s_hi) of the last sequence looked up kept
// by the caller: tokens of a thread advance monotonically, so cu_seqlens is
// read again only when a token leaves that sequence. Start with s_lo > s_hi.
__device__ __forceinline__ int first_key_cached(const int32_t* cu, int num_seqs, int window,
                                                int t, int& s_lo, int& s_hi) {
  if (t < s_lo || t >= s_hi) {
    const int s = seq_of_token(cu, num_seqs, t);
    s_lo = __ldg(cu + s);
    s_hi = __ldg(cu + s + 1);
  }
  return window > 0 ? max(s_lo, t - window + 1) : s_lo;
}

__device__ __forceinline__ int first_visible_key(const PrefillParams& p, int t) {
  return first_key(p.cu_seqlens, p.num_seqs, p.window, t);
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  constexpr int NCH = D / 64;  // 64-column (128-byte) chunks of the head dim
  constexpr uint32_t Q_CHUNK = 128 * 128;  // bytes of one 128-row x 128-byte chunk
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[3];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  // shared-memory carve-up (1024-byte aligned for the 128-byte swizzle atoms)
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t kv_chunk = static_cast<uint32_t>(p.BN) * 128u;
  const uint32_t sQ = base;
  const uint32_t sK = sQ + NCH * Q_CHUNK;
  const uint32_t sV = sK + NCH * kv_chunk;
  const uint32_t sP = sV + NCH * kv_chunk;
  const uint32_t bar_q = smem_u32(&bars[0]);
  const uint32_t bar_kv = smem_u32(&bars[1]);
  const uint32_t bar_mma = smem_u32(&bars[2]);

  // work unit: (token tile, kv head)
  const int tile = blockIdx.x / p.Hkv;
  const int g = blockIdx.x - tile * p.Hkv;
  const int tok_tile = p.reverse ? (p.n_tok_tiles - 1 - tile) : tile;
  const int t0 = tok_tile * p.TM;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv, 1);
    mbar_init(bar_mma, 1);
    abort_sh = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base_sh), p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort = &abort_sh;

  // ---- this thread's row -------------------------------------------------
  const int r = tid;
  const int tok_in_tile = r / p.G;
  const int hh = r - tok_in_tile * p.G;
  const int i = t0 + tok_in_tile;
  const int h = g * p.G + hh;
  const bool row_valid = (tok_in_tile < p.TM) && (i < p.total);
  int row_lo = 1, row_hi = 0;  // empty unless valid
  if (row_valid) {
    row_lo = first_visible_key(p, i);
    row_hi = i;
  }
  // keys of the whole tile: from the first key of its first token (the first
  // visible key never decreases along the packed axis) to its last token
  const int last_tok = min(t0 + p.TM, p.total) - 1;
  const int lo0 = first_visible_key(p, t0);
  const int nchunks = (last_tok - lo0 + p.BN) / p.BN;

  // Running max (log2 units) and two running denominators relative to it:
  // l_run sums P as rounded to bf16 for the PV product, so O / l_run is a
  // properly normalised average of what the MMA summed; l_lse sums P in fp32
  // for the LSE, so a dominant key's bf16 rounding does not reach the LSE.
  float m_run = -INFINITY;
  float l_run = 0.f, l_lse = 0.f;
  if (p.sink != nullptr && row_valid) {
    m_run = __ldg(p.sink + h) * kLog2e;
    l_run = 1.f;  // the sink term exp2(s - m) with m = s
    l_lse = 1.f;
  }

  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tS = tmem + lane_off;             // S: columns [0, BN)
  const uint32_t tO = tmem + lane_off + p.o_col;   // O: columns [o_col, o_col + D)
  const uint32_t idesc_s = idesc_bf16_f32(128, p.BN, false, false);
  const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_q, NCH * p.q_box_bytes);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
      tma_load_3d(sQ + ch * Q_CHUNK, &tm_q, bar_q, ch * 64, g * p.G, t0);
  }

  uint32_t mma_phase = 0;
  for (int c = 0; c < nchunks; ++c) {
    const int k0 = lo0 + c * p.BN;
    // ---- producer + MMA issue: load K/V chunk, S = Q K^T ------------------
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_kv, 2u * NCH * kv_chunk);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        tma_load_3d(sK + ch * kv_chunk, &tm_k, bar_kv, ch * 64, g, k0);
        tma_load_3d(sV + ch * kv_chunk, &tm_v, bar_kv, ch * 64, g, k0);
      }
      bool ok = true;
      if (c == 0) ok = mbar_wait(bar_q, 0, abort);
      ok = ok && mbar_wait(bar_kv, c & 1, abort);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;  // 16 columns = 32 bytes
          const uint64_t ad = smem_desc_sw128(sQ + (kk >> 2) * Q_CHUNK + koff, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sK + (kk >> 2) * kv_chunk + koff, 16, 1024);
          mma_bf16_ss(tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_mma);
      }
    }
    __syncwarp();
    if (!mbar_wait(bar_mma, mma_phase, abort)) break;
    mma_phase ^= 1;
    __syncwarp();  // tcgen05.ld below is warp-collective
    tc_fence_after();

    // ---- softmax pass 1: masked row max ------------------------------------
    const int cmin = row_lo - k0;  // visible columns [cmin, cmax]
    const int cmax = row_hi - k0;
    float mx = -INFINITY;
    for (int cb = 0; cb < p.BN; cb += 16) {
      uint32_t v[16];
      tmem_ld16(tS + cb, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int col = cb + e;
        if (col >= cmin && col <= cmax) mx = fmaxf(mx, __uint_as_float(v[e]));
      }
    }
    const float m_new = fmaxf(m_run, mx * p.scale_log2);
    const bool grow = m_new > m_run;
    const float alpha = grow ? ex2(m_run - m_new) : 1.f;  // ex2(-inf) = 0
    // rescale O in TMEM when some row's max grew (warp-uniform decision)
    if (c > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
      for (int db = 0; db < D; db += 16) {
        uint32_t v[16];
        tmem_ld16(tO + db, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
        tmem_st16(tO + db, v);
      }
      tmem_st_wait();
    }
    l_run *= alpha;
    l_lse *= alpha;
    m_run = m_new;

    // ---- softmax pass 2: P = exp2(x - m), row sum, P -> smem (bf16) --------
    const float mb = (m_run == -INFINITY) ? 0.f : m_run;
    float lsum = 0.f, lsum_f32 = 0.f;
    for (int cb = 0; cb < p.BN; cb += 16) {
      uint32_t v[16];
      tmem_ld16(tS + cb, v);
      tmem_ld_wait();
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const int col = cb + e;
        const float x0 = (col >= cmin && col <= cmax)
                             ? ex2(__uint_as_float(v[e]) * p.scale_log2 - mb) : 0.f;
        const float x1 = (col + 1 >= cmin && col + 1 <= cmax)
                             ? ex2(__uint_as_float(v[e + 1]) * p.scale_log2 - mb) : 0.f;
        w[e >> 1] = pack_bf16x2(x0, x1);
        lsum += bf16lo_to_f32(w[e >> 1]) + bf16hi_to_f32(w[e >> 1]);
        lsum_f32 += x0 + x1;
      }
      // K-major, 128-byte swizzle: row r, 16-byte unit u -> u ^ (r & 7)
      const uint32_t rowaddr = sP + (cb >> 6) * Q_CHUNK + r * 128;
      const uint32_t u0 = (cb & 63) >> 3;
      st_shared_v4(rowaddr + (((u0) ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
      st_shared_v4(rowaddr + (((u0 + 1) ^ (r & 7)) << 4), w[4], w[5], w[6], w[7]);
    }
    l_run += lsum;
    l_lse += lsum_f32;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V ------------------------------------------------------------
    if (tid == 0 && !*abort) {
      tc_fence_after();
      for (int kk = 0; kk < p.BN / 16; ++kk) {
        const uint64_t ad = smem_desc_sw128(sP + (kk >> 2) * Q_CHUNK + (kk & 3) * 32, 16, 1024);
        // V chunk as the MN-major B operand: 64-dim blocks kv_chunk apart
        // (LBO), 8-key groups 1024 bytes apart (SBO)
        const uint64_t bd = smem_desc_sw128(sV + kk * 2048, kv_chunk, 1024);
        mma_bf16_ss(tmem + p.o_col, ad, bd, idesc_pv, (c > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(bar_mma);
    }
    __syncwarp();
    if (!mbar_wait(bar_mma, mma_phase, abort)) break;
    mma_phase ^= 1;
    __syncwarp();  // tcgen05.ld below is warp-collective
    tc_fence_after();
  }

  // ---- epilogue: O / l -> bf16, LSE ------------------------------------------
  if (!*abort) {
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(i) * p.Hq + h) * D;
#pragma unroll
    for (int db = 0; db < D; db += 16) {
      uint32_t v[16];
      tmem_ld16(tO + db, v);
      tmem_ld_wait();
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2)
        w[e >> 1] = pack_bf16x2(__uint_as_float(v[e]) * inv_l, __uint_as_float(v[e + 1]) * inv_l);
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + db);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    if (row_valid && p.lse != nullptr)
      p.lse[static_cast<size_t>(h) * p.total + i] = (m_run + log2f(l_lse)) * kLn2;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace swa
