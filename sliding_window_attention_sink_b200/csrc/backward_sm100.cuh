// backward_sm100.cuh -- gradients of the sliding-window / global attention
// with a per-head sink: dq, dk, dv and the sink's gradient.
//
// Operation: the calculus of the forward of "MiMo-V2-Flash Technical Report"
// summary (mlpod.com), section 2.2.2 (the sink joins the softmax denominator
// and its max; it has no value). With p_ij = exp(scale q_i.k_j - lse_i) over
// the visible keys, p_sink,i = exp(s_h - lse_i), o_i = sum_j p_ij v_j and the
// output gradient dO:
//   Delta_i = dO_i . o_i
//   dS_ij   = p_ij (dO_i . v_j - Delta_i)
//   dq_i    = scale sum_j dS_ij k_j        dk_j = scale sum_i dS_ij q_i
//   dv_j    = sum_i p_ij dO_i              dsink_h = -sum_i p_sink,i Delta_i
// (the ICML talk write-up, hzrcw.cc, Q&A: the sink's gradient updates must
// stay stable at scale). K and V gradients of a kv head sum over its G query
// heads. P is recomputed from q, k and the forward's lse (fp32), as the
// forward computed it.
//
// Two launches:
//   bwd_dq_tc_kernel    persistent, warp-specialised, tcgen05: a tile is 128
//                       query rows (128/G tokens x the G heads of one kv head,
//                       as the forward packs them), resident with its dO rows;
//                       its epilogue warps first find Delta = dO . o for the
//                       next tile's rows (fp32, into the caller's workspace
//                       [Hq, total] for dk/dv) and add -exp(s - lse) Delta into
//                       dsink (zeroed by the call);
//                       the tile's keys [first key of its first token, its last
//                       token] stream in chunks of 64. Per chunk: S = Q K^T and
//                       dP = dO V^T (K-major operands, into TMEM), dS = P (dP -
//                       Delta) by the elementwise warps (thread = row), written
//                       back over S as bf16 pairs, then dQ += dS K (dS from TMEM,
//                       K MN-major). dQ accumulates in TMEM (two buffers: one
//                       tile drains while the next accumulates) and leaves as
//                       bf16 x scale;
//   bwd_dkdv_tc_kernel  persistent, warp-specialised, tcgen05: a tile is 128
//                       keys of one kv head, resident with their values; the
//                       query rows that see them (tokens [k0, last token that
//                       sees key k0 + 127) x the G heads) stream in blocks of 64
//                       rows (64/G tokens) with their lse and Delta (cp.async
//                       into the block's stage). Per block: S^T = K Q^T and dP^T
//                       = V dO^T (thread = key), P^T and dS^T written back over
//                       S^T and dP^T as bf16 pairs, then dV += P^T dO and dK +=
//                       dS^T Q (A from TMEM, dO and Q MN-major). dV and dK
//                       accumulate in TMEM across the tile's blocks.
//
// Roles of the two pipelines (15 warps, as in the chunked forward):
//   warps 0-7   two elementwise warpgroups; group hw takes score columns
//               [32 hw, 32 hw + 32) of the 64 and writes its 16 columns of
//               bf16 pairs over its own first 16 score columns, so the groups
//               never wait on each other;
//   warps 8-11  epilogue (TMEM accumulators -> bf16 -> global, one row each;
//               in dq also Delta and dsink, one tile ahead);
//   warp 12     producer (TMA; lse / Delta by cp.async for dk/dv);
//   warp 13     TMEM allocation; issues the two score MMAs;
//   warp 14     issues the accumulating MMAs.
// TMEM: score buffers b = 0, 1 at columns [128 b, 128 b + 64) (S or S^T) and
// [128 b + 64, 128 b + 128) (dP or dP^T); accumulators from column 256.
//
// About half of each (key tile x row block) of a sliding-window band is
// masked (M = 128 keys is the MMA's granularity), so the tensor work executed
// is about twice the algorithmic for W = 128. Every wait is bounded (mbar_wait)
// and a warp leaves its loop as one when a wait gives up; nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

struct BwdParams {
  const __nv_bfloat16 *q, *k, *v, *o, *dout;
  const float* lse;  // [Hq, total], natural log
  const int32_t* cu_seqlens;
  int num_seqs, total, Hq, Hkv, G, window;
  const float* sink;  // [Hq] or NULL
  float scale, scale_log2;
  float* delta;       // [Hq, total] (workspace)
  __nv_bfloat16 *dq, *dk, *dv;
  float* dsink;       // [Hq] or NULL; zeroed before the dq kernel
};

constexpr int kBtThreads = 480;  // 15 warps
constexpr int kBtQRows = 128;    // dq: query rows per tile
constexpr int kBtChunk = 64;     // dq: keys per chunk
constexpr int kBtKeys = 128;     // dk/dv: keys per tile
constexpr int kBtRows = 64;      // dk/dv: query rows per block
constexpr int kBtStages = 4;     // dk/dv: Q / dO block stages

struct BtParams {
  const int32_t* cu_seqlens;
  int num_seqs, total, Hq, Hkv, G, lg;  // lg = log2(G)
  int window;         // <= 0: the whole causal prefix
  int TM;             // dq: tokens per tile (128 / G)
  int TOK;            // dk/dv: tokens per block (64 / G)
  int n_units;        // dq: token tiles; dk/dv: key tiles
  int n_tiles;        // n_units * Hkv
  const float* lse;   // [Hq, total], natural log
  float* delta;       // [Hq, total]: written by dq, read by dk/dv
  const __nv_bfloat16 *o, *dout;  // dq: Delta = dout . o
  const float* sink;  // [Hq] or NULL
  float* dsink;       // [Hq] or NULL; zero before the dq kernel
  float scale, scale_log2;
  __nv_bfloat16 *dq, *dk, *dv;
  uint32_t q_box_bytes;  // dq: one 64-column box of a Q tile (128 rows)
};

// Dynamic shared memory (1 KB alignment slack included).
template <int D>
__host__ __device__ constexpr int bt_dq_kv_stages() { return D == 128 ? 3 : 4; }
template <int D>
__host__ __device__ inline size_t bt_dq_smem_bytes() {
  // two stages of (Q, dO) 128-row tiles; K/V stages of 64-key chunks
  return 1024 + 2 * 2 * (D / 64) * 16384 + bt_dq_kv_stages<D>() * 2 * (D / 64) * 8192;
}
template <int D>
__host__ __device__ inline size_t bt_dkdv_smem_bytes() {
  // one (K, V) 128-key tile; kBtStages of (Q, dO) 64-row blocks
  return 1024 + 2 * (D / 64) * 16384 + kBtStages * 2 * (D / 64) * 8192;
}

// cp.async completion counted on an mbarrier: one pending arrival of the
// barrier's expected count is taken by the thread's earlier cp.async copies.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}

// Accumulator rows (one per thread, 32 TMEM lanes per warp) -> bf16 x mul ->
// a global row of D values, in 32-column pieces. After the last TMEM load the
// warp's lane 0 arrives on `empty` (the accumulator may be overwritten).
template <int D>
__device__ __forceinline__ void bt_store_row(uint32_t tacc, float mul, __nv_bfloat16* row,
                                             bool valid, uint32_t empty, bool last, int lane) {
#pragma unroll
  for (int q = 0; q < D; q += 32) {
    uint32_t v[32];
    tmem_ld16_at(tacc + q, &v[0]);
    tmem_ld16_at(tacc + q + 16, &v[16]);
    tmem_ld_wait();
    if (last && q + 32 == D) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty);
    }
    if (valid) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* f = reinterpret_cast<const float*>(&v[u * 8]);
        uint4 w;
        w.x = pack_bf16x2(f[0] * mul, f[1] * mul);
        w.y = pack_bf16x2(f[2] * mul, f[3] * mul);
        w.z = pack_bf16x2(f[4] * mul, f[5] * mul);
        w.w = pack_bf16x2(f[6] * mul, f[7] * mul);
        *reinterpret_cast<uint4*>(row + q + u * 8) = w;
      }
    }
  }
}

// Every lane of the warp calls this with its own wait's outcome: true when all
// succeeded, so the warp leaves a loop together (its __syncwarp calls then
// always see all lanes).
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

// Column of the bf16-pair operand for k-step kk (16 score columns each) when
// group 0 wrote score columns [0, 32) into TMEM columns [0, 16) and group 1
// wrote [32, 64) into [32, 48).
__device__ __forceinline__ uint32_t bt_pair_col(int kk) {
  return static_cast<uint32_t>((kk >> 1) * 32 + (kk & 1) * 8);
}

// =========================================================================
// dq
// =========================================================================
template <int D>
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const BtParams p) {
  constexpr int NCH = D / 64;
  constexpr uint32_t QCH = 16384;  // 128 rows x 128 bytes
  constexpr uint32_t KCH = 8192;   // 64 keys x 128 bytes
  constexpr int NKV = bt_dq_kv_stages<D>();
  constexpr int HALF = kBtChunk / 2;
  constexpr uint32_t acc_col = 256;  // dQ buffers [256, 384) and [384, 512)
  extern __shared__ uint8_t bt_smem_q[];
  __shared__ __align__(8) uint64_t q_full[2], q_empty[2], kv_full[NKV], kv_empty[NKV];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], a_full[2], a_empty[2];
  // Delta of tile k's rows in slot k & 1, from the epilogue warps to the dS warps
  __shared__ __align__(8) uint64_t dl_full[2], dl_empty[2];
  __shared__ float delta_s[2][kBtQRows];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &abort_sh;

  const uint32_t base = (smem_u32(bt_smem_q) + 1023u) & ~1023u;
  const uint32_t sQ = base;                     // [stage][Q, dO][NCH] x QCH
  const uint32_t sK = sQ + 2 * 2 * NCH * QCH;   // [stage][K, V][NCH] x KCH
  auto q_addr = [&](int st, int which, int ch) -> uint32_t {
    return sQ + static_cast<uint32_t>((st * 2 + which) * NCH + ch) * QCH;
  };
  auto k_addr = [&](int st, int which, int ch) -> uint32_t {
    return sK + static_cast<uint32_t>((st * 2 + which) * NCH + ch) * KCH;
  };

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      // the S issuer's commit after a tile's last S, and the four epilogue
      // warps once they have read the tile's dO for Delta
      mbar_init(smem_u32(&q_empty[s]), 5);
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_empty[s]), 1);
      mbar_init(smem_u32(&p_full[s]), 8);
      mbar_init(smem_u32(&a_full[s]), 1);
      mbar_init(smem_u32(&a_empty[s]), 4);
      mbar_init(smem_u32(&dl_full[s]), 4);
      mbar_init(smem_u32(&dl_empty[s]), 8);
    }
    for (int s = 0; s < NKV; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
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

  // the k-th tile of this CTA: the last token tiles (most keys) first
  auto tile_of = [&](int k, int& g, int& tb) {
    const int f = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    const int rank = f / p.Hkv;
    g = f - rank * p.Hkv;
    tb = p.n_units - 1 - rank;
  };
  const int ntile = (p.n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                    static_cast<int>(gridDim.x);
  // keys of a tile: [lo, last token], chunks of 64
  auto tile_keys = [&](int tb, int& lo, int& nchunk) {
    const int t0 = tb * p.TM;
    const int t_last = min(t0 + p.TM, p.total) - 1;
    lo = first_key(p.cu_seqlens, p.num_seqs, p.window, t0);
    nchunk = (t_last - lo + kBtChunk) / kBtChunk;
  };

  if (warp < 8) {
    // ================= dS = P (dP - Delta), thread = row =====================
    const int hw = warp >> 2;
    const int r = 32 * (warp & 3) + lane;
    const int tok = r >> p.lg, hh = r - (tok << p.lg);
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    // this row's lse (log2 units), fetched one tile ahead
    auto row_lse = [&](int k) -> float {
      if (k >= ntile) return 0.f;
      int g, tb;
      tile_of(k, g, tb);
      const int i = tb * p.TM + tok;
      if (i >= p.total) return 0.f;
      return __ldg(p.lse + static_cast<size_t>(g * p.G + hh) * p.total + i) * kLog2e;
    };
    float l2_next = row_lse(0);
    int n = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const float l2 = l2_next;
      l2_next = row_lse(k + 1);
      // this row's Delta from the epilogue warps
      if (!warp_all(mbar_wait(smem_u32(&dl_full[k & 1]), (k >> 1) & 1, abort))) break;
      const float dl = delta_s[k & 1][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dl_empty[k & 1]));
      const int t0 = tb * p.TM;
      const int i = t0 + tok;
      int row_lo = 0, row_hi = -1;  // rows past the end see no key
      if (i < p.total) {
        row_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, i);
        row_hi = i;
      }
      const int t_last = min(t0 + p.TM, p.total) - 1;
      const int all_lo = first_key(p.cu_seqlens, p.num_seqs, p.window, t_last);
      const int all_hi = t0;
      const uint64_t nl2 = f2_pack(-l2, -l2);
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1;
        if (!warp_all(mbar_wait(smem_u32(&s_full[b]), (n >> 1) & 1, abort))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + b * 128 + hw * HALF;
        uint32_t s[HALF], d[HALF];
        tmem_ld16_at(tS, &s[0]);
        tmem_ld16_at(tS + 16, &s[16]);
        tmem_ld16_at(tS + 64, &d[0]);
        tmem_ld16_at(tS + 80, &d[16]);
        tmem_ld_wait();
        const int cb = lo + c * kBtChunk + hw * HALF;  // key of this group's column 0
        if (!(cb >= all_lo && cb + HALF - 1 <= all_hi)) {
          const int cmin = row_lo - cb, cmax = row_hi - cb;
#pragma unroll
          for (int e = 0; e < HALF; ++e)
            if (e < cmin || e > cmax) s[e] = 0xff800000u;  // -inf: P = 0
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < HALF; e += 2) {
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), sc2, nl2),
                    a0, a1);
          const float p0 = ex2(a0), p1 = ex2(a1);
          w[e >> 1] = pack_bf16x2(p0 * (__uint_as_float(d[e]) - dl),
                                  p1 * (__uint_as_float(d[e + 1]) - dl));
        }
        tmem_st16(tS, w);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[b]));
      }
    }
  } else if (warp < 12) {
    // ========= Delta (a tile ahead) and the epilogue: dQ x scale -> bf16 ======
    const int r = 32 * (warp & 3) + lane;
    const int tok = r >> p.lg, hh = r - (tok << p.lg);
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    // Delta = dO . o of this thread's row of tile k (fp32 over the bf16
    // values: o from global memory, all its loads in flight at once; dO from
    // the tile's Q stage, whose release waits for these reads) to slot k & 1
    // for the dS warps and to the workspace for dk/dv; dsink -= exp(s - lse)
    // Delta, summed over the warp's rows of each head (lanes with equal hh),
    // one atomic add per head and warp
    auto delta_of = [&](int k) -> bool {
      const int sl = k & 1;
      int g, tb;
      tile_of(k, g, tb);
      const int i = tb * p.TM + tok;
      const int h = g * p.G + hh;
      uint4 ov[D / 8];
      if (i < p.total) {
        const uint4* orow =
            reinterpret_cast<const uint4*>(p.o + (static_cast<size_t>(i) * p.Hq + h) * D);
#pragma unroll
        for (int u = 0; u < D / 8; ++u) ov[u] = __ldg(orow + u);
      }
      if (!warp_all(mbar_wait(smem_u32(&q_full[sl]), (k >> 1) & 1, abort) &&
                    mbar_wait(smem_u32(&dl_empty[sl]), ((k >> 1) & 1) ^ 1, abort)))
        return false;
      float dl = 0.f, ds = 0.f;
      if (i < p.total) {
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
          // dO row r, 16-byte unit u of the swizzled 64-column block u / 8
          uint32_t bv[4];
          ld_shared_v4(q_addr(sl, 1, u >> 3) + r * 128 + ((((u & 7) ^ (r & 7))) << 4), bv);
          const uint32_t av[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dl += bf16lo_to_f32(av[e]) * bf16lo_to_f32(bv[e]) +
                  bf16hi_to_f32(av[e]) * bf16hi_to_f32(bv[e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&q_empty[sl]));  // dO of this tile is read
      if (i < p.total) {
        const size_t idx = static_cast<size_t>(h) * p.total + i;
        p.delta[idx] = dl;
        if (p.sink != nullptr) ds = -expf(__ldg(p.sink + h) - __ldg(p.lse + idx)) * dl;
      }
      delta_s[sl][r] = dl;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&dl_full[sl]));
      if (p.dsink != nullptr && p.sink != nullptr) {
        // a warp's 32 rows: lane % G is the head within the group (G a power
        // of two); for G = 64 every lane has a head of its own
        for (int m = 16; m >= p.G; m >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, m);
        if (lane < p.G) atomicAdd(p.dsink + g * p.G + hh, ds);
      }
      return true;
    };
    bool ok = ntile == 0 || delta_of(0);
    for (int k = 0; k < ntile && ok && !*abort; ++k) {
      if (k + 1 < ntile && !delta_of(k + 1)) break;
      int g, tb;
      tile_of(k, g, tb);
      const int a = k & 1;
      if (!warp_all(mbar_wait(smem_u32(&a_full[a]), (k >> 1) & 1, abort))) break;
      __syncwarp();
      tc_fence_after();
      const int i = tb * p.TM + tok;
      const bool valid = i < p.total;
      __nv_bfloat16* row = p.dq + (static_cast<size_t>(valid ? i : 0) * p.Hq + g * p.G + hh) * D;
      bt_store_row<D>(tmem + lane_off + acc_col + a * 128, p.scale, row, valid,
                      smem_u32(&a_empty[a]), true, lane);
    }
  } else if (warp == 12) {
    // ============================ TMA producer ================================
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int n = 0;
      bool ok = true;
      for (int k = 0; k < ntile && ok; ++k) {
        int g, tb, lo, nchunk;
        tile_of(k, g, tb);
        tile_keys(tb, lo, nchunk);
        const int qs = k & 1;
        if (!mbar_wait(smem_u32(&q_empty[qs]), ((k >> 1) & 1) ^ 1, abort)) break;
        const uint32_t qbar = smem_u32(&q_full[qs]);
        mbar_arrive_expect_tx(qbar, 2 * NCH * p.q_box_bytes);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          tma_load_3d(q_addr(qs, 0, ch), &tm_q, qbar, ch * 64, g * p.G, tb * p.TM);
          tma_load_3d(q_addr(qs, 1, ch), &tm_do, qbar, ch * 64, g * p.G, tb * p.TM);
        }
        for (int c = 0; c < nchunk; ++c, ++n) {
          const int st = n % NKV;
          if (!mbar_wait(smem_u32(&kv_empty[st]), ((n / NKV) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          const uint32_t bar = smem_u32(&kv_full[st]);
          mbar_arrive_expect_tx(bar, 2 * NCH * KCH);
          const int key0 = lo + c * kBtChunk;
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            tma_load_3d(k_addr(st, 0, ch), &tm_k, bar, ch * 64, g, key0);
            tma_load_3d(k_addr(st, 1, ch), &tm_v, bar, ch * 64, g, key0);
          }
        }
      }
    }
  } else if (warp == 13) {
    // =================== S = Q K^T and dP = dO V^T ============================
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);
    const uint32_t idesc = idesc_bf16_f32(128, kBtChunk, false, false);
    int n = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const int qs = k & 1;
      if (!warp_all(mbar_wait(smem_u32(&q_full[qs]), (k >> 1) & 1, abort))) break;
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1, st = n % NKV;
        if (!warp_all(mbar_wait(smem_u32(&s_empty[b]), ((n >> 1) & 1) ^ 1, abort) &&
                      mbar_wait(smem_u32(&kv_full[st]), (n / NKV) & 1, abort))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t aq = kmaj | (q_addr(qs, 0, 0) >> 4);
        const uint64_t ado = kmaj | (q_addr(qs, 1, 0) >> 4);
        const uint64_t bk = kmaj | (k_addr(st, 0, 0) >> 4);
        const uint64_t bv = kmaj | (k_addr(st, 1, 0) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t offa = ((kk >> 2) * QCH + (kk & 3) * 32) >> 4;
            const uint32_t offb = ((kk >> 2) * KCH + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tmem + b * 128, aq + offa, bk + offb, idesc, kk > 0 ? 1u : 0u);
            mma_bf16_ss(tmem + b * 128 + 64, ado + offa, bv + offb, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&s_full[b]));
          if (c == nchunk - 1) mma_commit(smem_u32(&q_empty[qs]));
        }
        __syncwarp();
      }
    }
  } else if (warp == 14) {
    // ============================ dQ += dS K ==================================
    const uint32_t idesc = idesc_bf16_f32(128, D, false, true);
    // K as the MN-major B operand: 64-dim blocks KCH apart (LBO), 8-key groups
    // 1024 bytes apart (SBO)
    const uint64_t mnmaj = smem_desc_sw128(0, KCH, 1024);
    int n = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, tb, lo, nchunk;
      tile_of(k, g, tb);
      tile_keys(tb, lo, nchunk);
      const int a = k & 1;
      for (int c = 0; c < nchunk; ++c, ++n) {
        const int b = n & 1, st = n % NKV;
        if (!warp_all(mbar_wait(smem_u32(&p_full[b]), (n >> 1) & 1, abort) &&
                      (c > 0 || mbar_wait(smem_u32(&a_empty[a]), ((k >> 1) & 1) ^ 1, abort)))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t kd = mnmaj | (k_addr(st, 0, 0) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBtChunk / 16; ++kk)
            mma_bf16_ts(tmem + acc_col + a * 128, tmem + b * 128 + bt_pair_col(kk),
                        kd + ((kk * 16 * 128) >> 4), idesc, (c > 0 || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&s_empty[b]));
          mma_commit(smem_u32(&kv_empty[st]));
          if (c == nchunk - 1) mma_commit(smem_u32(&a_full[a]));
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =========================================================================
// dk, dv
// =========================================================================
template <int D>
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_do, const BtParams p) {
  constexpr int NCH = D / 64;
  constexpr uint32_t KCH = 16384;  // 128 keys x 128 bytes
  constexpr uint32_t RCH = 8192;   // 64 rows x 128 bytes
  constexpr int NS = kBtStages;
  constexpr int HALF = kBtRows / 2;
  constexpr uint32_t dv_col = 256, dk_col = 384;
  extern __shared__ uint8_t bt_smem_kv[];
  __shared__ __align__(8) uint64_t kv_full, kv_empty, qd_full[NS], qd_empty[NS];
  __shared__ __align__(8) uint64_t s_full[2], s_empty[2], p_full[2], a_full, a_empty;
  __shared__ __align__(16) float lse_s[NS][kBtRows], dlt_s[NS][kBtRows];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  volatile int* abort = &abort_sh;

  const uint32_t base = (smem_u32(bt_smem_kv) + 1023u) & ~1023u;
  const uint32_t sK = base;                    // [K, V][NCH] x KCH
  const uint32_t sQ = sK + 2 * NCH * KCH;      // [stage][Q, dO][NCH] x RCH
  auto r_addr = [&](int st, int which, int ch) -> uint32_t {
    return sQ + static_cast<uint32_t>((st * 2 + which) * NCH + ch) * RCH;
  };

  if (tid == 0) {
    mbar_init(smem_u32(&kv_full), 1);
    mbar_init(smem_u32(&kv_empty), 1);
    for (int s = 0; s < NS; ++s) {
      // the TMA arrival (with its bytes) and 32 cp.async completions
      mbar_init(smem_u32(&qd_full[s]), 33);
      mbar_init(smem_u32(&qd_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_empty[s]), 1);
      mbar_init(smem_u32(&p_full[s]), 8);
    }
    mbar_init(smem_u32(&a_full), 1);
    mbar_init(smem_u32(&a_empty), 4);
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

  // the k-th tile of this CTA: key tiles in order (under the causal mask the
  // first ones are seen by the most rows)
  auto tile_of = [&](int k, int& g, int& kt) {
    const int f = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
    kt = f / p.Hkv;
    g = f - kt * p.Hkv;
  };
  const int ntile = (p.n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                    static_cast<int>(gridDim.x);
  // one past the last token that sees key j (j < total)
  auto vis_end = [&](int j) -> int {
    const int s = seq_of_token(p.cu_seqlens, p.num_seqs, j);
    const int e = __ldg(p.cu_seqlens + s + 1);
    return (p.window > 0 && p.window < e - j) ? j + p.window : e;  // no overflow
  };
  // 64-row blocks of tile kt: tokens [k0, end of the last key's visibility)
  auto tile_blocks = [&](int kt) -> int {
    const int k0 = kt * kBtKeys;
    const int t_hi = vis_end(min(k0 + kBtKeys, p.total) - 1);
    return (t_hi - k0 + p.TOK - 1) / p.TOK;
  };

  if (warp < 8) {
    // ============ P^T and dS^T = P^T (dP^T - Delta), thread = key =============
    const int hw = warp >> 2;
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float sl2 = p.scale_log2;
    int m = 0;  // blocks done over this CTA's tiles
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, kt;
      tile_of(k, g, kt);
      (void)g;
      const int nblk = tile_blocks(kt);
      const int k0 = kt * kBtKeys;
      const int j = k0 + r;
      // tokens that see key j: [j, j_end)
      const int j_end = j < p.total ? vis_end(j) : j;
      for (int n = 0; n < nblk; ++n, ++m) {
        const int b = m & 1, st = m % NS;
        if (!warp_all(mbar_wait(smem_u32(&s_full[b]), (m >> 1) & 1, abort) &&
                      mbar_wait(smem_u32(&qd_full[st]), (m / NS) & 1, abort))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + b * 128 + hw * HALF;
        uint32_t s[HALF], d[HALF];
        tmem_ld16_at(tS, &s[0]);
        tmem_ld16_at(tS + 16, &s[16]);
        tmem_ld16_at(tS + 64, &d[0]);
        tmem_ld16_at(tS + 80, &d[16]);
        tmem_ld_wait();
        // column e is row 32 hw + e of the block, token t0 + ((32 hw + e) >> lg):
        // visible rows are [G (j - t0), G (j_end - t0)), token offsets clamped
        // to the block's [0, TOK]
        const int t0 = k0 + n * p.TOK;
        const int cmin = (min(max(j - t0, 0), p.TOK) << p.lg) - hw * HALF;
        const int cmax = (min(max(j_end - t0, 0), p.TOK) << p.lg) - 1 - hw * HALF;
        if (cmin > 0 || cmax < HALF - 1) {
#pragma unroll
          for (int e = 0; e < HALF; ++e)
            if (e < cmin || e > cmax) s[e] = 0xff800000u;  // -inf: P = 0
        }
        const float* ls = &lse_s[st][hw * HALF];
        const float* dls = &dlt_s[st][hw * HALF];
        uint32_t wp[16], wd[16];
#pragma unroll
        for (int e = 0; e < HALF; e += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(ls + e);
          const float4 d4 = *reinterpret_cast<const float4*>(dls + e);
          const float x0 = ex2(fmaf(__uint_as_float(s[e]), sl2, -l4.x * kLog2e));
          const float x1 = ex2(fmaf(__uint_as_float(s[e + 1]), sl2, -l4.y * kLog2e));
          const float x2 = ex2(fmaf(__uint_as_float(s[e + 2]), sl2, -l4.z * kLog2e));
          const float x3 = ex2(fmaf(__uint_as_float(s[e + 3]), sl2, -l4.w * kLog2e));
          wp[e >> 1] = pack_bf16x2(x0, x1);
          wp[(e >> 1) + 1] = pack_bf16x2(x2, x3);
          wd[e >> 1] = pack_bf16x2(x0 * (__uint_as_float(d[e]) - d4.x),
                                   x1 * (__uint_as_float(d[e + 1]) - d4.y));
          wd[(e >> 1) + 1] = pack_bf16x2(x2 * (__uint_as_float(d[e + 2]) - d4.z),
                                         x3 * (__uint_as_float(d[e + 3]) - d4.w));
        }
        tmem_st16(tS, wp);
        tmem_st16(tS + 64, wd);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[b]));
      }
    }
  } else if (warp < 12) {
    // ================= epilogue: dV, dK x scale -> bf16 =======================
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    for (int k = 0; k < ntile && !*abort; ++k) {
      int g, kt;
      tile_of(k, g, kt);
      if (!warp_all(mbar_wait(smem_u32(&a_full), k & 1, abort))) break;
      __syncwarp();
      tc_fence_after();
      const int j = kt * kBtKeys + r;
      const bool valid = j < p.total;
      const size_t off = (static_cast<size_t>(valid ? j : 0) * p.Hkv + g) * D;
      bt_store_row<D>(tmem + lane_off + dv_col, 1.f, p.dv + off, valid, 0u, false, lane);
      bt_store_row<D>(tmem + lane_off + dk_col, p.scale, p.dk + off, valid,
                      smem_u32(&a_empty), true, lane);
    }
  } else if (warp == 12) {
    // ==================== producer: TMA + lse / Delta =========================
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
    }
    int m = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, kt;
      tile_of(k, g, kt);
      const int nblk = tile_blocks(kt);
      const int k0 = kt * kBtKeys;
      // every lane waits; the warp leaves together if any wait gave up
      if (!warp_all(mbar_wait(smem_u32(&kv_empty), (k & 1) ^ 1, abort))) break;
      if (lane == 0) {
        const uint32_t bar = smem_u32(&kv_full);
        mbar_arrive_expect_tx(bar, 2 * NCH * KCH);
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          tma_load_3d(sK + ch * KCH, &tm_k, bar, ch * 64, g, k0);
          tma_load_3d(sK + (NCH + ch) * KCH, &tm_v, bar, ch * 64, g, k0);
        }
      }
      __syncwarp();
      for (int n = 0; n < nblk; ++n, ++m) {
        const int st = m % NS;
        if (!warp_all(mbar_wait(smem_u32(&qd_empty[st]), ((m / NS) & 1) ^ 1, abort))) {
          ok = false;
          break;
        }
        const int t0 = k0 + n * p.TOK;
        const uint32_t bar = smem_u32(&qd_full[st]);
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, 2 * NCH * RCH);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            tma_load_3d(r_addr(st, 0, ch), &tm_q, bar, ch * 64, g * p.G, t0);
            tma_load_3d(r_addr(st, 1, ch), &tm_do, bar, ch * 64, g * p.G, t0);
          }
        }
        // rows lane and lane + 32 of the block: lse and Delta (zero past the end)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rr = lane + 32 * u;
          const int t = t0 + (rr >> p.lg);
          const bool valid = t < p.total;
          const size_t idx =
              static_cast<size_t>(g * p.G + (rr & (p.G - 1))) * p.total + (valid ? t : 0);
          cp_async4_zfill(smem_u32(&lse_s[st][rr]), p.lse + idx, valid);
          cp_async4_zfill(smem_u32(&dlt_s[st][rr]), p.delta + idx, valid);
        }
        cp_async_mbar_arrive_noinc(bar);
        __syncwarp();
      }
    }
  } else if (warp == 13) {
    // ================= S^T = K Q^T and dP^T = V dO^T ==========================
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);
    const uint32_t idesc = idesc_bf16_f32(128, kBtRows, false, false);
    const uint64_t ak = kmaj | (sK >> 4);
    const uint64_t av = kmaj | ((sK + NCH * KCH) >> 4);
    int m = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, kt;
      tile_of(k, g, kt);
      const int nblk = tile_blocks(kt);
      if (!warp_all(mbar_wait(smem_u32(&kv_full), k & 1, abort))) break;
      for (int n = 0; n < nblk; ++n, ++m) {
        const int b = m & 1, st = m % NS;
        if (!warp_all(mbar_wait(smem_u32(&s_empty[b]), ((m >> 1) & 1) ^ 1, abort) &&
                      mbar_wait(smem_u32(&qd_full[st]), (m / NS) & 1, abort))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t bq = kmaj | (r_addr(st, 0, 0) >> 4);
        const uint64_t bd = kmaj | (r_addr(st, 1, 0) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t offa = ((kk >> 2) * KCH + (kk & 3) * 32) >> 4;
            const uint32_t offb = ((kk >> 2) * RCH + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tmem + b * 128, ak + offa, bq + offb, idesc, kk > 0 ? 1u : 0u);
            mma_bf16_ss(tmem + b * 128 + 64, av + offa, bd + offb, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&s_full[b]));
          if (n == nblk - 1) mma_commit(smem_u32(&kv_empty));
        }
        __syncwarp();
      }
    }
  } else if (warp == 14) {
    // ================= dV += P^T dO and dK += dS^T Q ==========================
    const uint32_t idesc = idesc_bf16_f32(128, D, false, true);
    // Q and dO as MN-major B operands: 64-dim blocks RCH apart (LBO), 8-row
    // groups 1024 bytes apart (SBO)
    const uint64_t mnmaj = smem_desc_sw128(0, RCH, 1024);
    int m = 0;
    bool ok = true;
    for (int k = 0; k < ntile && ok; ++k) {
      int g, kt;
      tile_of(k, g, kt);
      const int nblk = tile_blocks(kt);
      for (int n = 0; n < nblk; ++n, ++m) {
        const int b = m & 1, st = m % NS;
        if (!warp_all(mbar_wait(smem_u32(&p_full[b]), (m >> 1) & 1, abort) &&
                      (n > 0 || mbar_wait(smem_u32(&a_empty), (k & 1) ^ 1, abort)))) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t qd = mnmaj | (r_addr(st, 0, 0) >> 4);
        const uint64_t dd = mnmaj | (r_addr(st, 1, 0) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBtRows / 16; ++kk) {
            const uint32_t acol = bt_pair_col(kk);
            const uint32_t boff = (kk * 16 * 128) >> 4;
            const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_ts(tmem + dv_col, tmem + b * 128 + acol, dd + boff, idesc, acc);
            mma_bf16_ts(tmem + dk_col, tmem + b * 128 + 64 + acol, qd + boff, idesc, acc);
          }
          mma_commit(smem_u32(&qd_empty[st]));
          mma_commit(smem_u32(&s_empty[b]));
          if (n == nblk - 1) mma_commit(smem_u32(&a_full));
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
