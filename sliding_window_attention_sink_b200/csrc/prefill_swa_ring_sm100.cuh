// prefill_swa_ring_sm100.cuh -- sliding-window prefill as a persistent,
// warp-specialised pipeline on sm_100a.
//
// Operation: the same as prefill_sm100.cuh ("MiMo-V2-Flash Technical Report"
// summary, mlpod.com, section 2.2.2: the sink joins the softmax max and
// denominator; section 2.2.1: window of 128 tokens), for sliding windows whose
// whole key range for a tile fits one MMA (BN <= 256).
//
// Why a different kernel for SWA: with W = 128 a tile's keys are its own TM
// tokens plus the W - 1 before them, so consecutive tiles of one kv head share
// all but TM keys. Each CTA therefore walks a contiguous span of token tiles
// (all 148 SMs busy, one CTA each) and keeps K and V in a ring of TM-key
// blocks in shared memory: per tile it fetches one new block (TM keys) from
// HBM instead of the whole window. What remains per tile is the Q tile in and
// the O tile out -- the bytes that bound the layer -- and the pipeline below
// keeps them streaming:
//
//   warp 0      TMA producer: Q tile (3-D box [64, G, TM], NQ stages) and new
//               K/V blocks (box [64, 1, TM]) into the ring.
//   warp 1      TMEM allocation; one thread issues tcgen05.mma:
//               S = Q K^T into one of two TMEM S buffers (the window may wrap
//               around the ring: then two MMAs, N1 + N2 = BN), and
//               O = P V with P read from TMEM (TS form) and V from the ring.
//   warps 2-5   softmax: thread r owns TMEM lane r; masked max seeded with the
//               sink, P = exp2(x - m) written back over S as bf16 pairs; LSE.
//   warps 6-9   epilogue: O / l -> bf16 into a swizzled staging tile -> TMA
//               store.
//
// Every wait is bounded (see mbar_wait); nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kRingMaxBlocks = 16;
constexpr int kRingMaxQ = 4;

struct RingParams {
  const int32_t* cu_seqlens;
  int num_seqs;
  int total;
  int Hq, Hkv, G, TM;
  int window;
  int KB;       // key blocks before the diagonal block: ceil((W - 1) / TM)
  int NWIN;     // KB + 1 blocks per window; BN = NWIN * TM keys
  int NB;       // blocks in the ring (> NWIN)
  int NQ;       // Q stages
  int n_tok_tiles;
  int n_tiles;  // n_tok_tiles * Hkv
  const float* sink;
  float scale_log2;
  float* lse;
  uint32_t q_box_bytes;   // bytes of one 64-column Q box
  uint32_t s_stride;      // TMEM column of S / P buffer b is b * s_stride
  uint32_t o_col;         // TMEM column of O
};

// Smem bytes the ring kernel needs (1 KB alignment slack included).
__host__ __device__ inline size_t ring_smem_bytes(int D, int TM, int NB, int NQ) {
  const size_t nch = D / 64;
  return 1024 + static_cast<size_t>(NQ) * nch * 16384 + nch * 16384 +
         2 * nch * static_cast<size_t>(NB) * TM * 128;
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    prefill_swa_ring_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_o, const RingParams p) {
  constexpr int NCH = D / 64;
  constexpr uint32_t CH = 16384;  // one 128-row x 128-byte chunk
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full[kRingMaxQ], q_empty[kRingMaxQ];
  __shared__ __align__(8) uint64_t kv_full[kRingMaxBlocks], kv_empty[kRingMaxBlocks];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], l_free[2];
  __shared__ __align__(8) uint64_t o_full, o_empty;
  __shared__ float l_s[2][128];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &abort_sh;

  // ---- shared memory carve-up ---------------------------------------------
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t blk_bytes = static_cast<uint32_t>(p.TM) * 128u;   // one key block, one chunk
  const uint32_t ring_ch = static_cast<uint32_t>(p.NB) * blk_bytes; // one chunk of the ring
  const uint32_t sQ = base;                                        // NQ x NCH x CH
  const uint32_t sO = sQ + p.NQ * NCH * CH;                         // NCH x CH
  const uint32_t sK = sO + NCH * CH;                                // NCH x ring_ch
  const uint32_t sV = sK + NCH * ring_ch;

  // ---- this CTA's span of (kv head, token tile) pairs ---------------------
  const long long span_lo = static_cast<long long>(blockIdx.x) * p.n_tiles / gridDim.x;
  const long long span_hi = static_cast<long long>(blockIdx.x + 1) * p.n_tiles / gridDim.x;
  const int ntile = static_cast<int>(span_hi - span_lo);

  if (tid == 0) {
    for (int s = 0; s < p.NQ; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&q_empty[s]), 1);
    }
    for (int s = 0; s < p.NB; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&s_full[b]), 1);
      mbar_init(smem_u32(&s_empty[b]), 1);
      mbar_init(smem_u32(&p_full[b]), 4);
      mbar_init(smem_u32(&l_free[b]), 4);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), 4);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // tile index j (0..ntile-1) -> (g, tb); new blocks it brings into the ring
  auto tile_of = [&](int j, int& g, int& tb) {
    const long long f = span_lo + j;
    g = static_cast<int>(f / p.n_tok_tiles);
    tb = static_cast<int>(f - static_cast<long long>(g) * p.n_tok_tiles);
  };
  auto new_blocks = [&](int j) {
    if (j == 0) return p.NWIN;
    int g, tb;
    tile_of(j, g, tb);
    return tb == 0 ? p.NWIN : 1;  // a new kv head restarts the window
  };

  if (warp == 0) {
    // ======================= TMA producer ====================================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int nload = 0;
      for (int j = 0; j < ntile && !*abort; ++j) {
        int g, tb;
        tile_of(j, g, tb);
        const int st = j % p.NQ;
        if (!mbar_wait(smem_u32(&q_empty[st]), ((j / p.NQ) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(smem_u32(&q_full[st]), NCH * p.q_box_bytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_load_3d(sQ + (st * NCH + ch) * CH, &tm_q, smem_u32(&q_full[st]), ch * 64, g * p.G,
                      tb * p.TM);
        const int nnew = new_blocks(j);
        const int first_kb = tb - nnew + 1;  // absolute key block of the first new block
        for (int n = 0; n < nnew; ++n, ++nload) {
          const int slot = nload % p.NB;
          if (!mbar_wait(smem_u32(&kv_empty[slot]), ((nload / p.NB) & 1) ^ 1, abort)) break;
          const uint32_t bar = smem_u32(&kv_full[slot]);
          mbar_arrive_expect_tx(bar, 2u * NCH * blk_bytes);
          const int key0 = (first_kb + n) * p.TM;  // may be negative: zero fill
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            tma_load_3d(sK + ch * ring_ch + slot * blk_bytes, &tm_k, bar, ch * 64, g, key0);
            tma_load_3d(sV + ch * ring_ch + slot * blk_bytes, &tm_v, bar, ch * 64, g, key0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ======================================
    if (lane == 0) {
      const int BN = p.NWIN * p.TM;
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      int nload = 0;          // blocks loaded up to and including the current tile
      int win_first_prev = 0;
      // O = P V for tile j: P from TMEM (over S buffer j & 1), V from the ring
      auto issue_pv = [&](int j, int win_first) -> bool {
        const int b = j & 1;
        if (!mbar_wait(smem_u32(&p_full[b]), (j >> 1) & 1, abort)) return false;
        if (!mbar_wait(smem_u32(&o_empty), (j & 1) ^ 1, abort)) return false;
        tc_fence_after();
        for (int kk = 0; kk < BN / 16; ++kk) {
          const int wb = (kk * 16) / p.TM;       // block within the window
          const int off = kk * 16 - wb * p.TM;   // first key inside the block
          const int slot = (win_first + wb) % p.NB;
          // V as the MN-major B operand: 64-dim blocks ring_ch apart (LBO),
          // 8-key groups 1024 bytes apart (SBO)
          const uint64_t bd = smem_desc_sw128(sV + slot * blk_bytes + off * 128, ring_ch, 1024);
          mma_bf16_ts(tmem + p.o_col, tmem + b * p.s_stride + kk * 8, bd, idesc_pv,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&o_full));
        mma_commit(smem_u32(&s_empty[b]));
        return true;
      };
      for (int j = 0; j < ntile && !*abort; ++j) {
        const int b = j & 1, st = j % p.NQ;
        const int nnew = new_blocks(j);
        const int first_new = nload;
        nload += nnew;
        const int win_first = nload - p.NWIN;
        // A tile that starts a new kv head replaces the whole window: finish
        // the previous tile and release its blocks before waiting for the new
        // ones (the producer needs the slots).
        const bool restart = j > 0 && nnew == p.NWIN;
        if (restart) {
          if (!issue_pv(j - 1, win_first_prev)) break;
          for (int s = win_first_prev; s < first_new; ++s)
            mma_commit(smem_u32(&kv_empty[s % p.NB]));
        }
        if (!mbar_wait(smem_u32(&s_empty[b]), ((j >> 1) & 1) ^ 1, abort)) break;
        if (!mbar_wait(smem_u32(&q_full[st]), (j / p.NQ) & 1, abort)) break;
        bool ok = true;
        for (int s = first_new; s < nload && ok; ++s)
          ok = mbar_wait(smem_u32(&kv_full[s % p.NB]), (s / p.NB) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        // S = Q K^T over the window; two MMAs where it wraps around the ring
        const int slot0 = win_first % p.NB;
        const int n1 = min(p.NWIN, p.NB - slot0);  // blocks before the wrap
        const int n2 = p.NWIN - n1;
        const uint32_t idesc1 = idesc_bf16_f32(128, n1 * p.TM, false, false);
        const uint32_t idesc2 = idesc_bf16_f32(128, n2 > 0 ? n2 * p.TM : 16, false, false);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ch = kk >> 2, koff = (kk & 3) * 32;
          const uint64_t ad = smem_desc_sw128(sQ + (st * NCH + ch) * CH + koff, 16, 1024);
          const uint64_t bd1 =
              smem_desc_sw128(sK + ch * ring_ch + slot0 * blk_bytes + koff, 16, 1024);
          mma_bf16_ss(tmem + b * p.s_stride, ad, bd1, idesc1, kk > 0 ? 1u : 0u);
          if (n2 > 0) {
            const uint64_t bd2 = smem_desc_sw128(sK + ch * ring_ch + koff, 16, 1024);
            mma_bf16_ss(tmem + b * p.s_stride + n1 * p.TM, ad, bd2, idesc2, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(smem_u32(&s_full[b]));
        mma_commit(smem_u32(&q_empty[st]));
        // PV of the previous tile, then release the blocks the window left
        if (j > 0 && !restart) {
          if (!issue_pv(j - 1, win_first_prev)) break;
          for (int s = win_first_prev; s < win_first; ++s)
            mma_commit(smem_u32(&kv_empty[s % p.NB]));
        }
        win_first_prev = win_first;
      }
      if (ntile > 0 && !*abort) issue_pv(ntile - 1, win_first_prev);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ======================= softmax (warps 2..5) ============================
    const int r = 32 * (warp & 3) + lane;  // TMEM lane == tile row
    const int tok = r / p.G, hh = r - tok * p.G;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int BN = p.NWIN * p.TM;
    for (int j = 0; j < ntile; ++j) {
      int g, tb;
      tile_of(j, g, tb);
      const int b = j & 1;
      const int i = tb * p.TM + tok;
      const int h = g * p.G + hh;
      const bool valid = i < p.total;
      int row_lo = 1, row_hi = 0;  // empty unless valid
      if (valid) {
        row_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, i);
        row_hi = i;
      }
      const int kw0 = (tb - p.KB) * p.TM;  // key of S column 0
      const int cmin = row_lo - kw0, cmax = row_hi - kw0;
      const float sink2 = (valid && p.sink != nullptr) ? __ldg(p.sink + h) * kLog2e : -INFINITY;
      if (!mbar_wait(smem_u32(&s_full[b]), (j >> 1) & 1, abort)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + b * p.s_stride;
      // pass 1: masked row max, seeded with the sink
      float mx = -INFINITY;
      for (int cb = 0; cb < BN; cb += 16) {
        uint32_t v[16];
        tmem_ld16(tS + cb, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int col = cb + e;
          if (col >= cmin && col <= cmax) mx = fmaxf(mx, __uint_as_float(v[e]));
        }
      }
      const float m = fmaxf(sink2, mx * p.scale_log2);
      const float mb = (m == -INFINITY) ? 0.f : m;
      // pass 2: P = exp2(x - m) as bf16 pairs written over S (columns
      // [0, BN/2)); sums of the rounded P (for O) and of fp32 P (for LSE)
      float l_r = 0.f, l_x = 0.f;
      for (int cb = 0; cb < BN; cb += 16) {
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
          l_r += bf16lo_to_f32(w[e >> 1]) + bf16hi_to_f32(w[e >> 1]);
          l_x += x0 + x1;
        }
        tmem_st8(tS + (cb >> 1), w);
      }
      if (sink2 != -INFINITY) {
        const float ts = ex2(sink2 - mb);
        l_r += ts;
        l_x += ts;
      }
      tmem_st_wait();
      if (valid && p.lse != nullptr)
        p.lse[static_cast<size_t>(h) * p.total + i] = (mb + log2f(l_x)) * kLn2;
      // hand l to the epilogue once it has read this buffer's previous value
      if (!mbar_wait(smem_u32(&l_free[b]), ((j >> 1) & 1) ^ 1, abort)) break;
      l_s[b][r] = l_r;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[b]));
    }
  } else {
    // ======================= epilogue (warps 6..9) ===========================
    const int r = 32 * (warp & 3) + lane;
    const int et = tid - 192;  // 0..127
    const uint32_t tO = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + p.o_col;
    for (int j = 0; j < ntile; ++j) {
      int g, tb;
      tile_of(j, g, tb);
      const int b = j & 1;
      if (!mbar_wait(smem_u32(&o_full), j & 1, abort)) break;
      // p_full[b] of this tile completed before PV was issued; waiting on it
      // here orders the softmax's write of l_s[b] before the read below
      if (!mbar_wait(smem_u32(&p_full[b]), (j >> 1) & 1, abort)) break;
      __syncwarp();
      tc_fence_after();
      const float l = l_s[b][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_free[b]));
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      // the staging tile is free once the previous TMA store has read it
      if (et == 0) tma_store_wait_read<0>();
      named_bar_sync(1, 128);
#pragma unroll
      for (int db = 0; db < D; db += 16) {
        uint32_t v[16];
        tmem_ld16(tO + db, v);
        tmem_ld_wait();
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2)
          w[e >> 1] = pack_bf16x2(__uint_as_float(v[e]) * inv_l, __uint_as_float(v[e + 1]) * inv_l);
        // 128-byte swizzle, as the TMA store expects: unit u -> u ^ (r & 7)
        const uint32_t rowaddr = sO + (db >> 6) * CH + r * 128;
        const uint32_t u0 = (db & 63) >> 3;
        st_shared_v4(rowaddr + ((u0 ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
        st_shared_v4(rowaddr + (((u0 + 1) ^ (r & 7)) << 4), w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&o_empty));
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (et == 0) {
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          tma_store_3d(&tm_o, sO + ch * CH, ch * 64, g * p.G, tb * p.TM);
        tma_store_commit();
      }
    }
    if (et == 0) tma_store_wait_all<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
