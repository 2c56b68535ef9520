// prefill_swa_ring_sm100.cuh -- sliding-window prefill as a persistent,
// warp-specialised pipeline on sm_100a.
//
// Operation: the same as prefill_sm100.cuh ("MiMo-V2-Flash Technical Report"
// summary, mlpod.com, section 2.2.2: the sink joins the softmax max and
// denominator; section 2.2.1: window of 128 tokens), for sliding windows whose
// whole key range for a tile fits one MMA (BN <= 192).
//
// Why a different kernel for SWA: with W = 128 a tile's keys are its own TM
// tokens plus the W - 1 before them, so consecutive tiles of one kv head share
// all but TM keys. Each CTA therefore walks a contiguous span of token tiles
// (all SMs busy, one CTA each) and keeps K and V in a ring of TM-key blocks in
// shared memory: per tile it fetches one new block (TM keys) from HBM instead
// of the whole window. What remains per tile is the Q tile in and the O tile
// out -- the bytes that bound the layer -- and the pipeline below keeps them
// streaming:
//
//   warps 0-3   softmax warpgroup 0 and
//   warps 4-7   softmax warpgroup 1: both work on the same tile. Thread r of
//               each owns TMEM lane r (tile row r); warpgroup h takes S
//               columns [h*BN/2, (h+1)*BN/2) in one TMEM load into registers,
//               masks them (only 16-column chunks that cross some row's window
//               edge), and the two halves exchange their row maxima and sums
//               through shared memory. The max is seeded with the sink, the sum
//               gets the sink term; P = exp2(x - m) goes back over S as bf16
//               pairs (A operand of the PV MMA).
//   warps 8-11  epilogue: O / l -> bf16 into a swizzled staging tile -> TMA
//               store, one 64-column chunk at a time.
//   warp 12     TMA producer: Q tile (3-D box [64, G, TM], NQ stages) and new
//               K/V blocks (box [64, 1, TM]) into the ring.
//   warp 13     TMEM allocation; issues S = Q K^T (tcgen05.mma, K-major
//               operands) into S buffer (tile & 1); where the window wraps
//               around the ring, two MMAs per k-step (N1 + N2 = BN).
//   warp 14     issues O = P V (P from TMEM, V MN-major from the ring).
//
// S and PV have separate issuing warps because one thread issuing dependent
// tcgen05.mma back to back was measured at 90-230 cycles per instruction on
// B200 (more than the 64-72 cycles of tensor work of these N=128/144 shapes),
// while two issuers together reach the tensor rate.
//
// Every wait is bounded (see mbar_wait); nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"
#include "rope_sm100.cuh"

namespace swa {

// Pipeline timeline hooks: compiled out unless SWA_RING_TRACE is defined (a
// profiling build then supplies swa_ring_trace: clock64 stamps of one CTA,
// [role][tile][event], roles 0 producer, 1 S issuer, 2 PV issuer, 3 softmax,
// 4 epilogue; and swa_ring_cta_ns: globaltimer and clock64 at each CTA's start
// and end).
#ifdef SWA_RING_TRACE
__device__ unsigned long long* swa_ring_trace;
__device__ unsigned long long* swa_ring_cta_ns;
__device__ int swa_ring_trace_block;  // the CTA whose timeline is recorded
#define RING_CTA(ev)                                                                      \
  do {                                                                                    \
    if (threadIdx.x == 0) {                                                               \
      swa_ring_cta_ns[blockIdx.x * 4 + (ev)] = globaltimer_ns();                          \
      swa_ring_cta_ns[blockIdx.x * 4 + 2 + (ev)] = static_cast<unsigned long long>(clock64()); \
      unsigned smid_;                                                                     \
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid_));                                  \
      swa_ring_cta_ns[160 * 4 + blockIdx.x] = smid_;                                      \
    }                                                                                     \
  } while (0)
#define RING_TRACE(role, j, ev)                                                           \
  do {                                                                                    \
    if (blockIdx.x == swa_ring_trace_block && (j) < 128)                                 \
      swa_ring_trace[((role) * 128 + (j)) * 8 + (ev)] = static_cast<unsigned long long>(clock64()); \
  } while (0)
#else
#define RING_TRACE(role, j, ev) \
  do {                          \
  } while (0)
#define RING_CTA(ev) \
  do {               \
  } while (0)
#endif

constexpr int kRingMaxBlocks = 16;
constexpr int kRingMaxQ = 4;
constexpr int kRingThreads = 480;  // 15 warps
constexpr int kRingMaxBN16 = 12;   // BN <= 192: a half row fits in registers
constexpr int kRingRanges = 4;     // tile ranges queued between the producer and the rest
constexpr int kRingRangeReaders = 14;  // warps other than the producer

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
  // Tile schedule. Tiles f = g * n_tok_tiles + tb are taken in ranges of
  // consecutive f, one range per work unit u: units u < n_static are the
  // static share [u * static_tiles, (u + 1) * static_tiles); unit
  // n_static + d is the range of dyn_span tiles from dyn_base + d * dyn_span.
  // A CTA first does unit blockIdx.x. Then, with sched == NULL (the grid has
  // one CTA per unit), it takes over units of CTAs that have not started yet
  // by cancelling their launch (cluster launch control); with a sched
  // counter (the grid has n_static CTAs), it draws d from sched[0], and
  // sched[1] counts finished CTAs, the last of which sets both back to zero.
  unsigned int* sched;
  int n_static;
  int static_tiles;
  int dyn_base;
  int dyn_span;
};

// Smem bytes the ring kernel needs (1 KB alignment slack included).
__host__ __device__ inline size_t ring_smem_bytes(int D, int TM, int NB, int NQ) {
  const size_t nch = D / 64;
  return 1024 + static_cast<size_t>(NQ) * nch * 16384 + nch * 16384 +
         2 * nch * static_cast<size_t>(NB) * TM * 128;
}

// BN16 = BN / 16 is fixed at compile time so a half row of scores lives in
// registers.
//
// ROPE: q and k arrive before the rotary embedding. The epilogue warpgroup
// rotates each Q tile in its stage and each new K block in its ring slot (in
// shared memory, in place, rounded to bf16) before the S issuer may use them
// (barriers q_rot / k_rot instead of the TMA barriers), then drains the
// previous tile's O: per tile it does rotate(j), drain(j - 1). Thread item
// (token, 8-pair group) computes the group's 8 angles once and rotates the G
// query rows of that token and the token's key row (the tile's own key block
// holds the tile's tokens). For the last ring_W tokens of each sequence it
// also writes the rotated key row and the value row into the caller's ring.
template <int D, int BN16, bool ROPE>
__global__ void __launch_bounds__(kRingThreads, 1)
    prefill_swa_ring_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_o, const RingParams p,
                            const __grid_constant__ RopeArgs rope) {
  constexpr int NCH = D / 64;
  constexpr uint32_t CH = 16384;  // one 128-row x 128-byte chunk
  constexpr int BN = BN16 * 16;
  constexpr int HALF = BN / 2;    // S columns per warpgroup (a multiple of 8)
  constexpr int H16 = HALF / 16;  // x16 TMEM loads per half row ...
  constexpr int H8 = (HALF % 16) / 8;  // ... plus one x8 load when HALF % 16 == 8
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full[kRingMaxQ], q_empty[kRingMaxQ];
  __shared__ __align__(8) uint64_t kv_full[kRingMaxBlocks], kv_empty[kRingMaxBlocks];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], l_free[2];
  __shared__ __align__(8) uint64_t o_full, o_empty;
  // ROPE only: Q stage / K block rotated in place
  __shared__ __align__(8) uint64_t q_rot[kRingMaxQ], k_rot[kRingMaxBlocks];
  __shared__ float red_max[2][128], red_lr[2][128], red_lx[2][128], l_s[2][128];
  // ranges of tiles, from the producer to the 14 other warps
  __shared__ __align__(8) uint64_t rq_full[kRingRanges], rq_empty[kRingRanges];
  __shared__ int rq_lo[kRingRanges], rq_hi[kRingRanges];
  // cluster launch control: the response to a cancellation request
  __shared__ __align__(16) uint32_t clc_resp[4];
  __shared__ __align__(8) uint64_t clc_bar;
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
      mbar_init(smem_u32(&p_full[b]), 8);
      mbar_init(smem_u32(&l_free[b]), 4);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), 4);
    for (int q = 0; q < kRingRanges; ++q) {
      mbar_init(smem_u32(&rq_full[q]), 1);
      mbar_init(smem_u32(&rq_empty[q]), kRingRangeReaders);
    }
    mbar_init(smem_u32(&clc_bar), 1);
    if (ROPE) {
      for (int s = 0; s < p.NQ; ++s) mbar_init(smem_u32(&q_rot[s]), 4);
      for (int s = 0; s < p.NB; ++s) mbar_init(smem_u32(&k_rot[s]), 4);
    }
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
  RING_CTA(0);

  // tile f -> (kv head g, token tile tb)
  auto tile_of = [&](int f, int& g, int& tb) {
    g = f / p.n_tok_tiles;
    tb = f - g * p.n_tok_tiles;
  };
  // key blocks tile tb brings into the ring: the whole window at the start of
  // a range or of a kv head, else one
  auto new_blocks = [&](bool range_start, int tb) { return range_start || tb == 0 ? p.NWIN : 1; };
  // the q-th range of this CTA (every warp but the producer reads each one);
  // false at the end of the schedule or when a wait gave up
  auto next_range = [&](int q, int& f0, int& f1) -> bool {
    const int s = q % kRingRanges;
    if (!mbar_wait(smem_u32(&rq_full[s]), (q / kRingRanges) & 1, abort)) return false;
    f0 = rq_lo[s];
    f1 = rq_hi[s];
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&rq_empty[s]));
    return f0 < f1;
  };

  if (warp < 8) {
    // ================== softmax (two warpgroups, one tile) ===================
    const int hw = warp >> 2;              // half of the row
    const int r = 32 * (warp & 3) + lane;  // TMEM lane == tile row
    const int tok = r / p.G, hh = r - tok * p.G;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    // sequence bounds of this row's token and of the tile's last token, and
    // this row's sink, carried from tile to tile
    int row_s_lo = 1, row_s_hi = 0, last_s_lo = 1, last_s_hi = 0;
    int sink_g = -1;
    float sink_h = -INFINITY;
    int j = 0;  // tiles done by this CTA: buffer parities
    bool stop = false;
    for (int q = 0; !stop; ++q) {
     int f0 = 0, f1 = 0;
     // every softmax thread leaves together (a named barrier follows)
     if (named_bar_any(1, 256, !next_range(q, f0, f1))) break;
     for (int f = f0; f < f1; ++f, ++j) {
      int g, tb;
      tile_of(f, g, tb);
      const int b = j & 1;
      const int t0 = tb * p.TM;
      const int i = t0 + tok;
      const int h = g * p.G + hh;
      const bool valid = i < p.total;
      int row_lo = 1, row_hi = 0;  // empty unless valid
      if (valid) {
        row_lo = first_key_cached(p.cu_seqlens, p.num_seqs, p.window, i, row_s_lo, row_s_hi);
        row_hi = i;
      }
      const int c0 = (tb - p.KB) * p.TM + hw * HALF;  // key of this half's column 0
      // visible columns of this half: e with (e - cmin) in [0, span]
      const int cmin = row_lo - c0;
      const unsigned span = static_cast<unsigned>(row_hi - row_lo);
      // columns visible to every valid row of the tile (uniform): from the
      // last valid token's first key to the first token itself
      const int t_last = min(t0 + p.TM, p.total) - 1;
      const int all_lo =
          first_key_cached(p.cu_seqlens, p.num_seqs, p.window, t_last, last_s_lo, last_s_hi) - c0;
      const int all_hi = t0 - c0;
      if (g != sink_g) {  // the sink changes with the kv head only
        sink_g = g;
        sink_h = p.sink != nullptr ? __ldg(p.sink + h) * kLog2e : -INFINITY;
      }
      const float sink2 = valid ? sink_h : -INFINITY;
      if (tid == 0) RING_TRACE(3, j, 0);
      const bool s_ok = mbar_wait(smem_u32(&s_full[b]), (j >> 1) & 1, abort);
      __syncwarp();
      tc_fence_after();
      if (tid == 0) RING_TRACE(3, j, 1);
      const uint32_t tS = tmem + lane_off + b * p.s_stride;
      uint32_t v[HALF];
#pragma unroll
      for (int c = 0; c < H16; ++c) tmem_ld16_at(tS + hw * HALF + c * 16, &v[c * 16]);
      if (H8) tmem_ld8_at(tS + hw * HALF + H16 * 16, &v[H16 * 16]);
      tmem_ld_wait();
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < HALF; c += 16) {
        const int n = (HALF - c) >= 16 ? 16 : 8;
        if (!(c >= all_lo && c + n - 1 <= all_hi)) {  // some row's window edge is here
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (e < n && static_cast<unsigned>(c + e - cmin) > span) v[c + e] = 0xff800000u;
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          if (e < n) {
            mx0 = max3(mx0, __uint_as_float(v[c + e]), __uint_as_float(v[c + e + 1]));
            mx1 = max3(mx1, __uint_as_float(v[c + e + 2]), __uint_as_float(v[c + e + 3]));
          }
        }
      }
      const float mx = fmaxf(mx0, mx1);
      red_max[hw][r] = mx;
      if (tid == 0) RING_TRACE(3, j, 2);
      // both halves have read S: P may go over it. A failed wait anywhere
      // stops every softmax thread here.
      tc_fence_before();
      if (named_bar_any(1, 256, !s_ok || *abort != 0)) {
        stop = true;
        break;
      }
      tc_fence_after();
      if (tid == 0) RING_TRACE(3, j, 3);
      const float m = fmaxf(sink2, fmaxf(mx, red_max[hw ^ 1][r]) * p.scale_log2);
      const float mb = (m == -INFINITY) ? 0.f : m;
      // P = exp2(x - m) (masked: exp2(-inf) = 0) as bf16 pairs over S
      // columns [hw*HALF/2, (hw+1)*HALF/2); sums of the rounded P (for O)
      // and of fp32 P (for the LSE)
      uint64_t lr2 = 0, lx2 = 0;  // packed pair sums (0.0f, 0.0f)
      const uint64_t nm2 = f2_pack(-mb, -mb);
      const uint32_t tP = tS + hw * (HALF / 2);
#pragma unroll
      for (int c = 0; c < HALF; c += 16) {
        uint32_t w[8];
        const int n = (HALF - c) >= 16 ? 16 : 8;
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          if (e < n) {
            float t0f, t1f;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(v[c + e]), __uint_as_float(v[c + e + 1])),
                             sc2, nm2),
                      t0f, t1f);
            const float x0 = ex2(t0f), x1 = ex2(t1f);
            w[e >> 1] = pack_bf16x2(x0, x1);
            lr2 = f2_add(lr2, f2_pack(bf16lo_to_f32(w[e >> 1]), bf16hi_to_f32(w[e >> 1])));
            lx2 = f2_add(lx2, f2_pack(x0, x1));
          }
        }
        if (n == 16) tmem_st8(tP + c / 2, w);
        else tmem_st4(tP + c / 2, w);
      }
      {
        float a0, a1;
        f2_unpack(lr2, a0, a1);
        red_lr[hw][r] = a0 + a1;
        f2_unpack(lx2, a0, a1);
        red_lx[hw][r] = a0 + a1;
      }
      tmem_st_wait();
      tc_fence_before();
      if (tid == 0) RING_TRACE(3, j, 4);
      named_bar_sync(1, 256);
      if (tid == 0) RING_TRACE(3, j, 5);
      float l_x = 0.f;
      if (hw == 0) {
        float l_r = red_lr[0][r] + red_lr[1][r];
        l_x = red_lx[0][r] + red_lx[1][r];
        if (sink2 != -INFINITY) {
          const float ts = ex2(sink2 - mb);
          l_r += ts;
          l_x += ts;
        }
        // l for the epilogue, once it has read this buffer's previous value
        // (on a failed wait the next tile's barrier stops the loop)
        if (mbar_wait(smem_u32(&l_free[b]), ((j >> 1) & 1) ^ 1, abort)) l_s[b][r] = l_r;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&p_full[b]));
      if (tid == 0) RING_TRACE(3, j, 6);
      if (hw == 0 && valid && p.lse != nullptr)
        p.lse[static_cast<size_t>(h) * p.total + i] = (mb + lg2(l_x)) * kLn2;
     }
    }
  } else if (warp < 12) {
    // ======================= epilogue (warps 8..11) ==========================
    const int r = 32 * (warp & 3) + lane;
    const bool issuer = tid == 256;
    const uint32_t tO = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + p.o_col;
    // O of tile jd (kv head gd, token tile tbd) to HBM; false when a wait gave
    // up (the epilogue warps then leave together)
    auto drain = [&](int jd, int gd, int tbd) -> bool {
      const int b = jd & 1;
      if (issuer) RING_TRACE(4, jd, 0);
      // p_full[b] of this tile completed before PV was issued; waiting on it
      // too orders the softmax's write of l_s[b] before the read below
      const bool ok = mbar_wait(smem_u32(&o_full), jd & 1, abort) &&
                      mbar_wait(smem_u32(&p_full[b]), (jd >> 1) & 1, abort);
      if (named_bar_any(2, 128, !ok)) return false;
      if (issuer) RING_TRACE(4, jd, 1);
      __syncwarp();
      tc_fence_after();
      const float l = l_s[b][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_free[b]));
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      // O leaves one 64-column chunk at a time: TMEM -> registers -> bf16 ->
      // staging chunk (128-byte swizzle: 16-byte unit u of row r at u ^ (r&7))
      // -> TMA store as its own bulk group. The staging chunk is reused once
      // its previous store has read it. TMEM O is released after the last
      // chunk's load. The chunk loop stays rolled (smaller code: the roles
      // share each SM sub-partition's instruction cache).
#pragma unroll 1
      for (int ch = 0; ch < NCH; ++ch) {
        uint32_t v[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16) tmem_ld16_at(tO + ch * 64 + c, &v[c]);
        tmem_ld_wait();
        if (ch == NCH - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&o_empty));
          if (issuer) RING_TRACE(4, jd, 2);
        }
        if (issuer) tma_store_wait_read<NCH - 1>();
        named_bar_sync(2, 128);
        const uint32_t rowaddr = sO + ch * CH + r * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(v[u * 8 + 2 * e]) * inv_l,
                               __uint_as_float(v[u * 8 + 2 * e + 1]) * inv_l);
          st_shared_v4(rowaddr + ((u ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(2, 128);
        if (issuer) {
          tma_store_3d(&tm_o, sO + ch * CH, ch * 64, gd * p.G, tbd * p.TM);
          tma_store_commit();
        }
      }
      if (issuer) RING_TRACE(4, jd, 3);
      return true;
    };
    int j = 0;
    bool stop = false;
    if constexpr (!ROPE) {
      for (int q = 0; !stop; ++q) {
        int f0 = 0, f1 = 0;
        if (named_bar_any(2, 128, !next_range(q, f0, f1))) break;
        for (int f = f0; f < f1; ++f, ++j) {
          int g, tb;
          tile_of(f, g, tb);
          if (!drain(j, g, tb)) {
            stop = true;
            break;
          }
        }
      }
    } else {
      constexpr int NK = D / 16;  // 8-pair groups per row
      const bool inter = rope.interleaved != 0;
      // cached sequence of the last token looked up
      int s_lo = 1, s_hi = 0, s_idx = 0, s_p0 = 0;
      // unit u of row `row` in a 1024-byte-aligned 128-byte-swizzled block
      auto unit_addr = [](uint32_t blk, int row, int u) -> uint32_t {
        return blk + row * 128 + ((u ^ (row & 7)) << 4);
      };
      // rotate tile jr's Q stage and its new K blocks [first_new, last_new)
      auto rotate = [&](int jr, int first_new, int last_new, int gr, int tbr) -> bool {
        const int st = jr % p.NQ;
        bool ok = mbar_wait(smem_u32(&q_full[st]), (jr / p.NQ) & 1, abort);
        for (int s = first_new; s < last_new && ok; ++s)
          ok = mbar_wait(smem_u32(&kv_full[s % p.NB]), (s / p.NB) & 1, abort);
        if (named_bar_any(2, 128, !ok)) return false;
        const int t0 = tbr * p.TM;
        const int nnew = last_new - first_new;
        const int first_kb = tbr - nnew + 1;
        const uint32_t qst = sQ + st * NCH * CH;
        const uint32_t kslot = static_cast<uint32_t>((last_new - 1) % p.NB) * blk_bytes;
        for (int it = r; it < p.TM * NK; it += 128) {
          const int tok = it / NK, k = it - tok * NK;
          int da, db;
          rope_units<D>(k, inter, da, db);
          const int cha = da >> 6, ua = (da & 63) >> 3, chb = db >> 6, ub = (db & 63) >> 3;
          float cs[8], sn[8];
          uint32_t a[4], bq[4];
          const int t = t0 + tok;
          if (t < p.total) {
            const int ps = rope_token_pos(p.cu_seqlens, p.num_seqs, rope.pos0, t, s_lo, s_hi,
                                          s_idx, s_p0);
            rope_cos_sin8(rope, ps, 8 * k, cs, sn);
            // the token's G query rows
            for (int hh = 0; hh < p.G; ++hh) {
              const int row = tok * p.G + hh;
              const uint32_t aa = unit_addr(qst + cha * CH, row, ua);
              const uint32_t ab = unit_addr(qst + chb * CH, row, ub);
              ld_shared_v4(aa, a);
              ld_shared_v4(ab, bq);
              rope_rotate8(a, bq, cs, sn, inter);
              st_shared_v4(aa, a[0], a[1], a[2], a[3]);
              st_shared_v4(ab, bq[0], bq[1], bq[2], bq[3]);
            }
            // its key row in the tile's own (last new) block
            const uint32_t ka = unit_addr(sK + cha * ring_ch + kslot, tok, ua);
            const uint32_t kb = unit_addr(sK + chb * ring_ch + kslot, tok, ub);
            ld_shared_v4(ka, a);
            ld_shared_v4(kb, bq);
            rope_rotate8(a, bq, cs, sn, inter);
            st_shared_v4(ka, a[0], a[1], a[2], a[3]);
            st_shared_v4(kb, bq[0], bq[1], bq[2], bq[3]);
            if (rope.k_ring != nullptr && t - s_lo >= (s_hi - s_lo) - rope.ring_W) {
              const size_t rrow = (static_cast<size_t>(s_idx) * rope.ring_W +
                                   static_cast<size_t>(ps) % rope.ring_W) * p.Hkv + gr;
              __nv_bfloat16* kr = rope.k_ring + rrow * D;
              __nv_bfloat16* vr = rope.v_ring + rrow * D;
              st_global_v4(kr + da, a);
              st_global_v4(kr + db, bq);
              ld_shared_v4(unit_addr(sV + cha * ring_ch + kslot, tok, ua), a);
              ld_shared_v4(unit_addr(sV + chb * ring_ch + kslot, tok, ub), bq);
              st_global_v4(vr + da, a);
              st_global_v4(vr + db, bq);
            }
          }
          // earlier blocks of a window loaded whole (range or kv-head start)
          for (int n = 0; n + 1 < nnew; ++n) {
            const int tk = (first_kb + n) * p.TM + tok;
            if (tk < 0 || tk >= p.total) continue;  // zero fill
            const int ps = rope_token_pos(p.cu_seqlens, p.num_seqs, rope.pos0, tk, s_lo, s_hi,
                                          s_idx, s_p0);
            rope_cos_sin8(rope, ps, 8 * k, cs, sn);
            const uint32_t sl = static_cast<uint32_t>((first_new + n) % p.NB) * blk_bytes;
            const uint32_t ka = unit_addr(sK + cha * ring_ch + sl, tok, ua);
            const uint32_t kb = unit_addr(sK + chb * ring_ch + sl, tok, ub);
            ld_shared_v4(ka, a);
            ld_shared_v4(kb, bq);
            rope_rotate8(a, bq, cs, sn, inter);
            st_shared_v4(ka, a[0], a[1], a[2], a[3]);
            st_shared_v4(kb, bq[0], bq[1], bq[2], bq[3]);
          }
        }
        // the rotated tiles go to the tensor cores (async proxy)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&q_rot[st]));
          for (int s = first_new; s < last_new; ++s) mbar_arrive(smem_u32(&k_rot[s % p.NB]));
        }
        return true;
      };
      int nload = 0;
      int pj = -1, pg = 0, ptb = 0;  // the tile whose O is still to drain
      for (int q = 0; !stop; ++q) {
        int f0 = 0, f1 = 0;
        if (named_bar_any(2, 128, !next_range(q, f0, f1))) break;
        for (int f = f0; f < f1; ++f, ++j) {
          int g, tb;
          tile_of(f, g, tb);
          const int first_new = nload;
          nload += new_blocks(f == f0, tb);
          if (!rotate(j, first_new, nload, g, tb) || (pj >= 0 && !drain(pj, pg, ptb))) {
            stop = true;
            break;
          }
          pj = j;
          pg = g;
          ptb = tb;
        }
      }
      if (!stop && pj >= 0) drain(pj, pg, ptb);
    }
    if (issuer) tma_store_wait_all<0>();
  } else if (warp == 12) {
    // ================= TMA producer and tile scheduler ======================
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
      int nload = 0, j = 0, q = 0;
      // hand range [f0, f1) to the other warps as the q-th; f0 >= f1 ends
      auto publish = [&](int f0, int f1) -> bool {
        const int s = q % kRingRanges;
        if (!mbar_wait(smem_u32(&rq_empty[s]), ((q / kRingRanges) & 1) ^ 1, abort)) return false;
        rq_lo[s] = f0;
        rq_hi[s] = f1;
        mbar_arrive(smem_u32(&rq_full[s]));
        ++q;
        return true;
      };
      bool ok = true;
      uint32_t clc_phase = 0;
      int u = static_cast<int>(blockIdx.x);  // this CTA's own unit first
      for (int k = 0; ok && !*abort; ++k) {
        if (k > 0) {
          if (p.sched != nullptr) {  // the next unit from the counter
            u = p.n_static + static_cast<int>(atomicAdd(p.sched, 1u));
          } else {  // the unit of a CTA whose launch this request cancels
            mbar_arrive_expect_tx(smem_u32(&clc_bar), 16u);
            clc_try_cancel(smem_u32(clc_resp), smem_u32(&clc_bar));
            if (!mbar_wait(smem_u32(&clc_bar), clc_phase, abort)) break;
            clc_phase ^= 1u;
            if (!clc_query(smem_u32(clc_resp), u)) break;  // none left
          }
        }
        int f0, f1;
        if (u < p.n_static) {
          f0 = u * p.static_tiles;
          f1 = min(f0 + p.static_tiles, p.n_tiles);
        } else {
          const long long s0 =
              p.dyn_base + static_cast<long long>(u - p.n_static) * p.dyn_span;
          f0 = static_cast<int>(min(s0, static_cast<long long>(p.n_tiles)));
          f1 = min(f0 + p.dyn_span, p.n_tiles);
        }
        if (f0 >= f1) {
          // an empty static share: go on to the other units; past the end of
          // the counter's ranges: done
          if (k > 0 && p.sched != nullptr) break;
          continue;
        }
        if (!publish(f0, f1)) break;
        for (int f = f0; f < f1 && ok; ++f, ++j) {
          int g, tb;
          tile_of(f, g, tb);
          const int st = j % p.NQ;
          RING_TRACE(0, j, 0);
          if (!mbar_wait(smem_u32(&q_empty[st]), ((j / p.NQ) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          RING_TRACE(0, j, 1);
          mbar_arrive_expect_tx(smem_u32(&q_full[st]), NCH * p.q_box_bytes);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_3d(sQ + (st * NCH + ch) * CH, &tm_q, smem_u32(&q_full[st]), ch * 64,
                        g * p.G, tb * p.TM);
          const int nnew = new_blocks(f == f0, tb);
          const int first_kb = tb - nnew + 1;  // absolute key block of the first new block
          for (int n = 0; n < nnew; ++n, ++nload) {
            const int slot = nload % p.NB;
            if (!mbar_wait(smem_u32(&kv_empty[slot]), ((nload / p.NB) & 1) ^ 1, abort)) {
              ok = false;
              break;
            }
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
      publish(0, 0);  // end of the schedule
      // with a counter: this CTA draws no more ranges; the last CTA to get
      // here clears the call's scheduler slot for the next call that uses it
      if (p.sched != nullptr) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
          __threadfence();
          atomicExch(p.sched, 0u);
          atomicExch(p.sched + 1, 0u);
        }
      }
    }
  } else if (warp == 13) {
    // ======================= S = Q K^T issuer ================================
    // Descriptors are computed by the whole warp; one elected lane issues.
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);  // layout bits, no address
    int nload = 0, j = 0;
    bool stop = false;
    for (int q = 0; !stop; ++q) {
     int f0 = 0, f1 = 0;
     if (!next_range(q, f0, f1)) break;
     for (int f = f0; f < f1; ++f, ++j) {
      int g, tb;
      tile_of(f, g, tb);
      const int b = j & 1, st = j % p.NQ;
      const int first_new = nload;
      nload += new_blocks(f == f0, tb);
      const int win_first = nload - p.NWIN;
      if (lane == 0) RING_TRACE(1, j, 0);
      if (!mbar_wait(smem_u32(&s_empty[b]), ((j >> 1) & 1) ^ 1, abort)) {
        stop = true;
        break;
      }
      if (lane == 0) RING_TRACE(1, j, 1);
      // with ROPE, Q and the new K blocks once the epilogue has rotated them
      if (!mbar_wait(smem_u32(ROPE ? &q_rot[st] : &q_full[st]), (j / p.NQ) & 1, abort)) {
        stop = true;
        break;
      }
      if (lane == 0) RING_TRACE(1, j, 2);
      bool ok = true;
      for (int s = first_new; s < nload && ok; ++s)
        ok = mbar_wait(smem_u32(ROPE ? &k_rot[s % p.NB] : &kv_full[s % p.NB]), (s / p.NB) & 1,
                       abort);
      if (!ok) {
        stop = true;
        break;
      }
      if (lane == 0) RING_TRACE(1, j, 3);
      __syncwarp();
      tc_fence_after();
      // the window's blocks are consecutive ring slots; two MMAs per k-step
      // where they wrap
      const int slot0 = win_first % p.NB;
      const int n1 = min(p.NWIN, p.NB - slot0);
      const int n2 = p.NWIN - n1;
      const uint32_t idesc1 = idesc_bf16_f32(128, n1 * p.TM, false, false);
      const uint32_t idesc2 = idesc_bf16_f32(128, n2 > 0 ? n2 * p.TM : 16, false, false);
      const uint32_t dS = tmem + b * p.s_stride;
      const uint32_t dS2 = dS + n1 * p.TM;
      const uint64_t aq = kmaj | ((sQ + st * NCH * CH) >> 4);
      const uint64_t bk1 = kmaj | ((sK + slot0 * blk_bytes) >> 4);
      const uint64_t bk2 = kmaj | (sK >> 4);
      const bool leader = elect_one();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * CH + (kk & 3) * 32) >> 4;
        const uint32_t offk = ((kk >> 2) * ring_ch + (kk & 3) * 32) >> 4;
        if (leader) {
          mma_bf16_ss(dS, aq + off, bk1 + offk, idesc1, kk > 0 ? 1u : 0u);
          if (n2 > 0) mma_bf16_ss(dS2, aq + off, bk2 + offk, idesc2, kk > 0 ? 1u : 0u);
        }
      }
      if (leader) {
        mma_commit(smem_u32(&s_full[b]));
        mma_commit(smem_u32(&q_empty[st]));
        RING_TRACE(1, j, 4);
      }
      __syncwarp();
     }
    }
  } else if (warp == 14) {
    // ======================= O = P V issuer ==================================
    const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
    // V as the MN-major B operand: 64-dim blocks ring_ch apart (LBO), 8-key
    // groups 1024 bytes apart (SBO)
    const uint64_t mnmaj = smem_desc_sw128(0, ring_ch, 1024);
    const uint32_t ring_keys = static_cast<uint32_t>(p.NB * p.TM);
    int nload = 0, j = 0;
    bool stop = false;
    for (int q = 0; !stop; ++q) {
     int f0 = 0, f1 = 0;
     if (!next_range(q, f0, f1)) break;
     for (int f = f0; f < f1; ++f, ++j) {
      int g, tb;
      tile_of(f, g, tb);
      const int b = j & 1;
      nload += new_blocks(f == f0, tb);
      const int win_first = nload - p.NWIN;
      // first window block of the next tile (blocks before it are released):
      // one block on within a range and a kv head, else the window restarts
      const bool next_slides = f + 1 < f1 && tb + 1 < p.n_tok_tiles;
      const int win_next = next_slides ? win_first + 1 : nload;
      if (lane == 0) RING_TRACE(2, j, 0);
      if (!mbar_wait(smem_u32(&p_full[b]), (j >> 1) & 1, abort)) {
        stop = true;
        break;
      }
      if (lane == 0) RING_TRACE(2, j, 1);
      if (!mbar_wait(smem_u32(&o_empty), (j & 1) ^ 1, abort)) {
        stop = true;
        break;
      }
      if (lane == 0) RING_TRACE(2, j, 2);
      __syncwarp();
      tc_fence_after();
      // key k of the window sits in ring row (first_row + k) mod ring_keys
      uint32_t row = static_cast<uint32_t>((win_first % p.NB) * p.TM);
      const uint32_t aP = tmem + b * p.s_stride;  // P: 8 columns per 16 keys
      const bool leader = elect_one();
#pragma unroll
      for (int kk = 0; kk < BN16; ++kk) {
        const uint64_t bd = mnmaj | ((sV + row * 128) >> 4);
        if (leader) mma_bf16_ts(tmem + p.o_col, aP + kk * 8, bd, idesc_pv, kk > 0 ? 1u : 0u);
        row += 16;
        if (row >= ring_keys) row -= ring_keys;
      }
      if (leader) {
        mma_commit(smem_u32(&o_full));
        mma_commit(smem_u32(&s_empty[b]));
        for (int s = win_first; s < win_next; ++s) mma_commit(smem_u32(&kv_empty[s % p.NB]));
        RING_TRACE(2, j, 3);
      }
      __syncwarp();
     }
    }
  }

  tc_fence_before();
  __syncthreads();
  RING_CTA(1);
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
