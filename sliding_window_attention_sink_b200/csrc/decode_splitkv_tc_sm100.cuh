// decode_splitkv_tc_sm100.cuh -- the split-KV decode over a long KV cache
// (the global-attention layers) on the tcgen05 tensor cores: the persistent
// design of decode_tc_sm100.cuh, with an online softmax over the steps of a
// range.
//
// Operation (decode_splitkv_sm100.cuh has the cache convention and the
// merge): the sink attention of the "MiMo-V2-Flash Technical Report" summary,
// section 2.2.2, at decode over the global layers of section 2.2, with the MTP
// drafts of section 2.3; each (sequence, range of cached positions, kv head)
// writes a partial state (O unnormalised, m, l_r, l_x) that
// decode_split_combine_kernel merges. It replaced an mma.sync kernel with one
// CTA per range (0.183 ms against 0.150 ms for the global-layer decode
// workload).
//
// Design (sm_100a). A unit is one (sequence, range, kv head). Its cached
// positions go through in steps of 128 (two 64-position tiles of the ring;
// W is a multiple of 64, so a tile never wraps), the last range's new tokens
// as one more step of 16 keys.
// * One CTA per SM; the grid has one CTA per unit, and the CTAs that run take
//   over the units of CTAs that have not started (cluster launch control), as
//   in decode_tc_sm100.cuh. The producer hands the units (with the sequence's
//   position) to the other warps through a ring in shared memory.
// * S = Q K^T of a step is an M = 64 tcgen05 MMA with the 32 query rows spread
//   over the four TMEM lane quarters (the Q descriptor steps 512 bytes per
//   8-row group); S is double-buffered in TMEM, so the next step's S runs
//   while this one's softmax does.
// * One group of four softmax warps (8 rows each, 4 threads per row, 16-lane
//   x 256-bit loads) keeps the running max of each row, with a lazy rescale:
//   the reference max moves only when a step's max exceeds it by more than
//   2^8 (log2 units); O in TMEM and the row sums are then rescaled by the
//   threads that own the row, once the previous step's P V has completed. P is
//   written over S (16 x 128b) and O += P V accumulates in TMEM over the
//   range's steps.
// * Four epilogue warps write the partial state once the unit's last P V is
//   done. A unit with no cached position and no new token never enters the
//   unit ring: the producer marks its state empty (m = -inf, which the merge
//   skips). In the ring, long runs of such units (the last ranges of short
//   sequences) would let the producer fill it and block before a load that the
//   ring's slowest reader, the epilogue, is waiting for.
// * V rows a step's MMA uses but no position of the range owns (past the end
//   of the range, the new-token step's padding, stale or never-initialised
//   shared memory) are zeroed before P is released: P is 0 there, and 0 * V
//   must stay 0.
// * Warps: 0-3 softmax, 4-7 epilogue, 8 MMA issuer and TMEM owner, 9 TMA
//   producer.
// Every wait is bounded (mbar_wait); a wait that gives up sets the abort flag
// and the device error bit and every role leaves its loop.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_splitkv_sm100.cuh"
#include "decode_tc_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kSplTcWarps = 10;
constexpr int kSplTcThreads = kSplTcWarps * 32;
constexpr int kSplTcStep = 128;     // cached positions per step (two tiles)
constexpr int kSplTcKSlots = 3;     // K slots
constexpr int kSplTcVSlots = 2;     // V slots
constexpr int kSplTcQSlots = 2;     // Q slots (one per unit in flight)
// readers of a unit-ring entry: the MMA warp, 4 softmax and 4 epilogue warps
constexpr int kSplTcReaders = 9;
constexpr float kSplTcRescale = 8.f;  // lazy-rescale threshold (log2 units)

// Dynamic shared memory: Q slots [D/64][32][128], K and V slots
// [D/64][128 rows][128 bytes], 1 KB of alignment slack. The S MMA's A operand
// reads up to 4608 bytes from a Q chunk's start, past the Q slots into the K
// slots.
__host__ __device__ inline size_t split_tc_smem_bytes(int D) {
  const size_t nch = static_cast<size_t>(D / 64);
  return 1024 + nch * (kSplTcQSlots * 4096 + (kSplTcKSlots + kSplTcVSlots) * 128 * 128);
}

template <int D>
__global__ void __launch_bounds__(kSplTcThreads, 1)
    decode_split_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kc,
                           const __grid_constant__ CUtensorMap tm_vc,
                           const __grid_constant__ CUtensorMap tm_kn,
                           const __grid_constant__ CUtensorMap tm_vn, const SplitParams p) {
  constexpr int NCH = D / 64;
  constexpr int T = kSplitTile;                // 64 positions per ring tile
  constexpr uint32_t SLOT = NCH * 128 * 128;   // one K or V slot
  constexpr uint32_t S_COLS = 128;             // TMEM columns of one S buffer
  constexpr uint32_t O_COL = 2 * S_COLS;
  extern __shared__ uint8_t spl_smem[];
  __shared__ __align__(8) uint64_t q_full[kSplTcQSlots], q_empty[kSplTcQSlots];
  __shared__ __align__(8) uint64_t k_full[kSplTcKSlots], k_empty[kSplTcKSlots];
  __shared__ __align__(8) uint64_t v_full[kSplTcVSlots], v_empty[kSplTcVSlots];
  __shared__ __align__(8) uint64_t s_full[2], s_free[2], p_full[2];
  __shared__ __align__(8) uint64_t o_full, o_empty, l_full, l_free;
  __shared__ __align__(8) uint64_t ur_full[kDecTcUnits], ur_empty[kDecTcUnits];
  __shared__ int ring_u[kDecTcUnits], ring_P[kDecTcUnits];  // unit (-1: none) and position
  __shared__ __align__(16) uint32_t clc_resp[4];
  __shared__ __align__(8) uint64_t clc_bar;
  __shared__ float l_m[32], l_r_s[32], l_x_s[32];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int W = p.W, n_q = p.n_q, G = p.G, R = p.R;
  const uint32_t base = (smem_u32(spl_smem) + 1023u) & ~1023u;
  const uint32_t sQ = base;                                   // Q slots
  const uint32_t sK = sQ + kSplTcQSlots * NCH * 4096;         // K slots
  const uint32_t sV = sK + kSplTcKSlots * SLOT;               // V slots

  if (tid == 0) {
    for (int s = 0; s < kSplTcQSlots; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&q_empty[s]), 1);
    }
    for (int s = 0; s < kSplTcKSlots; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_free[s]), 1);
      mbar_init(smem_u32(&p_full[s]), 4);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), 4);
    mbar_init(smem_u32(&l_full), 4);
    mbar_init(smem_u32(&l_free), 4);
    for (int s = 0; s < kDecTcUnits; ++s) {
      mbar_init(smem_u32(&ur_full[s]), 1);
      mbar_init(smem_u32(&ur_empty[s]), kSplTcReaders);
    }
    mbar_init(smem_u32(&clc_bar), 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  auto wait_all = [&](uint64_t& bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar), parity, abort));
  };
  // unit u -> (sequence b, range s, kv head g): CTAs that run together take
  // the same positions of all kv heads of a sequence
  auto unit_of = [&](int u, int& b, int& s, int& g) {
    const int bs = u / p.Hkv;
    g = u - bs * p.Hkv;
    b = bs / p.S;
    s = bs - b * p.S;
  };
  // the unit's range of cached positions [r0, r1), its first tile start t0,
  // its tiles and steps (the last range adds the new-token step)
  struct Range { int r0, r1, t0, ntile, ncached, nsteps; bool last; };
  auto range_of = [&](int s, int P) -> Range {
    Range rg;
    const int lo0 = max(0, P - W + 1);
    rg.r0 = lo0 + s * p.chunk;
    rg.r1 = min(rg.r0 + p.chunk, P);
    rg.t0 = (rg.r0 / T) * T;
    rg.ntile = rg.r1 > rg.r0 ? (rg.r1 - rg.t0 + T - 1) / T : 0;
    rg.ncached = (rg.ntile + 1) / 2;
    rg.last = s == p.S - 1;
    rg.nsteps = rg.ncached + (rg.last ? 1 : 0);
    return rg;
  };
  // entry i of the unit ring, read by a whole warp, which then releases it
  auto read_unit = [&](int i, int& u, int& P) -> bool {
    const int e = i % kDecTcUnits;
    if (!wait_all(ur_full[e], (i / kDecTcUnits) & 1)) return false;
    u = ring_u[e];
    P = ring_P[e];
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ur_empty[e]));
    return true;
  };

  if (warp < 4) {
    // ============ softmax (4 warps, 8 rows each, every step) =================
    const int q4 = warp;
    const int s4 = lane & 3;
    const int r = 8 * q4 + (lane >> 2);  // query row (TMEM lane 32*q4 + lane/4)
    const bool rvalid = r < R;
    const int t = rvalid ? r / G : -1;
    const uint32_t lq = static_cast<uint32_t>(32 * q4) << 16;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    int n = 0;       // steps over this CTA's units: S buffer n & 1, V slot n % 2
    int handed = 0;  // units with steps whose row state went to the epilogue
    bool ok = true;
    for (int i = 0; ok; ++i) {
      int u = -1, P = 0;
      if (!read_unit(i, u, P) || u < 0) break;
      int b, s, g;
      unit_of(u, b, s, g);
      const Range rg = range_of(s, P);
      // first cached position this row sees in the range (invalid rows none)
      const int vlo = rvalid ? max(rg.r0, max(0, P + t - W + 1)) : 0x7fffffff;
      float m_used = -INFINITY;  // reference max of P (log2 units)
      float l_r = 0.f, l_x = 0.f;
      for (int k = 0; k < rg.nsteps; ++k, ++n) {
        const int bb = n & 1;
        const bool cached = k < rg.ncached;
        const int pos0 = rg.t0 + k * kSplTcStep;  // position of column 0 (cached steps)
        // this thread's invisible 8-key blocks: keys 8k' + 2*s4 + e
        uint32_t inv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          auto blocks = [&](int x0, int x1) -> uint32_t {
            const int k0 = min(16, max(0, (x0 - 2 * s4 - e + 7) >> 3));
            const int k1 = min(16, max(0, (x1 - 2 * s4 - e + 7) >> 3));
            return k1 > k0 ? (1u << k1) - (1u << k0) : 0u;
          };
          if (cached)  // visible: positions [vlo, r1)
            inv[e] = blocks(0, vlo - pos0) | blocks(rg.r1 - pos0, 128);
          else         // new tokens 0 .. t
            inv[e] = blocks(t + 1, 128);
        }
        if (!wait_all(s_full[bb], (n >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tS = tmem + lq + static_cast<uint32_t>(bb) * S_COLS;
        uint32_t v[64];
#pragma unroll
        for (int m = 0; m < 4; ++m) tmem_ld_16x256b_x4(tS + 32 * m, &v[16 * m]);
        tmem_ld_wait();
        float mx = -INFINITY;
#pragma unroll
        for (int kb = 0; kb < 16; ++kb) {
          v[4 * kb] = ((inv[0] >> kb) & 1u) ? 0xff800000u : v[4 * kb];
          v[4 * kb + 1] = ((inv[1] >> kb) & 1u) ? 0xff800000u : v[4 * kb + 1];
          mx = max3(mx, __uint_as_float(v[4 * kb]), __uint_as_float(v[4 * kb + 1]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float cm = mx * p.scale_log2;
        // lazy rescale: the reference moves only when the max outgrows it
        const bool grow = cm > m_used + kSplTcRescale;
        if (__any_sync(0xffffffffu, grow)) {
          const float m_new = grow ? cm : m_used;
          const float alpha = grow ? ex2(m_used - m_new) : 1.f;  // exp2(-inf) = 0
          // O holds the P V of this unit's earlier steps once P V(n - 1) has
          // completed (its commit frees S buffer (n - 1) & 1)
          if (k > 0) {
            if (!wait_all(s_free[(n - 1) & 1], ((n - 1) >> 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tO = tmem + lq + O_COL;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t w[16];
              tmem_ld_16x256b_x4(tO + 32 * c, w);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
              tmem_st_16x256b_x4(tO + 32 * c, w);
            }
            tmem_st_wait();
          }
          l_r *= alpha;
          l_x *= alpha;
          m_used = m_new;
        }
        const float mb = (m_used == -INFINITY) ? 0.f : m_used;
        // P = exp2(x - m_used) as bf16 pairs over S
        uint64_t lr2 = 0, lx2 = 0;
        const uint64_t nm2 = f2_pack(-mb, -mb);
        uint32_t w[16];
#pragma unroll
        for (int kb = 0; kb < 16; ++kb) {
          float t0f, t1f;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[4 * kb]), __uint_as_float(v[4 * kb + 1])),
                           sc2, nm2),
                    t0f, t1f);
          const float x0 = ex2(t0f), x1 = ex2(t1f);
          const uint32_t pk = pack_bf16x2(x0, x1);
          w[kb] = pk;
          lr2 = f2_add(lr2, f2_pack(bf16lo_to_f32(pk), bf16hi_to_f32(pk)));
          lx2 = f2_add(lx2, f2_pack(x0, x1));
        }
        tmem_st_16x128b_x8_dup(tS, &w[0]);
        tmem_st_16x128b_x8_dup(tS + 32, &w[8]);
        {
          float a0, a1;
          f2_unpack(lr2, a0, a1);
          l_r += a0 + a1;
          f2_unpack(lx2, a0, a1);
          l_x += a0 + a1;
        }
        // V rows the MMA uses that no position of the range owns: zeros
        {
          const int vb = n & 1;
          const int used = cached ? 128 : 16;
          const int valid = cached ? max(0, min(128, rg.r1 - pos0)) : n_q;
          if (valid < used) {
            if (!wait_all(v_full[vb], (n >> 1) & 1)) {
              ok = false;
              break;
            }
            const uint32_t vs = sV + static_cast<uint32_t>(vb) * SLOT;
            const int per = (used - valid) * 8;  // 16-byte units per chunk
            for (int idx = lane + 32 * q4; idx < NCH * per; idx += 128) {
              const int ch = idx / per, rem = idx - ch * per;
              st_shared_zero16(vs + ch * 128 * 128 + (valid + (rem >> 3)) * 128 + (rem & 7) * 16);
            }
            fence_proxy_async_smem();
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[bb]));
      }
      if (!ok) break;
      // the unit's row state for the epilogue (sums over the row's 4 threads)
      l_r += __shfl_xor_sync(0xffffffffu, l_r, 1);
      l_x += __shfl_xor_sync(0xffffffffu, l_x, 1);
      l_r += __shfl_xor_sync(0xffffffffu, l_r, 2);
      l_x += __shfl_xor_sync(0xffffffffu, l_x, 2);
      if (rg.nsteps > 0) {
        if (!wait_all(l_free, (handed & 1) ^ 1)) break;
        if (s4 == 0) {
          l_m[r] = m_used;
          l_r_s[r] = l_r;
          l_x_s[r] = l_x;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&l_full));
        ++handed;
      }
    }
  } else if (warp < 8) {
    // ============ epilogue (4 warps): the partial state of each unit =========
    const int q4 = warp & 3;
    const int s4 = lane & 3;
    const int r = 8 * q4 + (lane >> 2);
    const uint32_t tO = tmem + (static_cast<uint32_t>(32 * q4) << 16) + O_COL;
    int done = 0;  // units with steps drained (o_full / l_full parities)
    for (int i = 0;; ++i) {
      int u = -1, P = 0;
      if (!read_unit(i, u, P) || u < 0) break;
      int b, s, g;
      unit_of(u, b, s, g);
      const Range rg = range_of(s, P);
      (void)rg;  // every unit in the ring has a step
      const int unit = (b * p.Hkv + g) * p.S + s;  // partial-state slot
      float* orow = p.part + (static_cast<size_t>(unit) * 32 + r) * (D + 4);
      // l_full precedes o_full's wait: the softmax hands l over after its
      // last P, before the last P V completes
      if (!wait_all(l_full, done & 1) || !wait_all(o_full, done & 1)) break;
      tc_fence_after();
      const float m = l_m[r], lr = l_r_s[r], lx = l_x_s[r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_free));
      uint32_t o[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_16x256b_x4(tO + 32 * c, &o[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&o_empty));
#pragma unroll
      for (int c = 0; c < D / 8; ++c)
        *reinterpret_cast<float2*>(orow + 8 * c + 2 * s4) =
            make_float2(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]));
      if (s4 == 0) {
        orow[D] = m;
        orow[D + 1] = lr;
        orow[D + 2] = lx;
      }
      ++done;
    }
  } else if (warp == 8) {
    // ======================= MMA issuer ======================================
    // Over the CTA's steps n: S(n) = Q K^T, then O += P V of step n - 1.
    const uint64_t amaj = smem_desc_sw128(0, 16, 512);   // Q: 8-row groups 512 B apart
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);  // K: K-major
    const uint64_t mnmaj = smem_desc_sw128(0, NCH > 1 ? 128 * 128 : 16, 1024);  // V: MN-major
    const uint32_t idesc_pv = idesc_bf16_f32(64, D, false, true);
    int n = 0;          // steps issued
    int units_o = 0;    // units with steps whose O has been started (also their Q slot)
    // the step before n: its buffer, whether it began / ended its unit, its keys
    bool prev = false, prev_first = false, prev_last = false;
    int prev_keys = 0;
    int prev_o = 0;
    bool ok = true;
    auto issue_pv = [&]() -> bool {
      const int j = n - 1, bb = j & 1;
      if (!wait_all(p_full[bb], (j >> 1) & 1)) return false;
      if (!wait_all(v_full[bb], (j >> 1) & 1)) return false;
      if (prev_first && !wait_all(o_empty, (prev_o & 1) ^ 1)) return false;
      tc_fence_after();
      const uint32_t aP = tmem + static_cast<uint32_t>(bb) * S_COLS;  // P: 8 columns per 16 keys
      const uint32_t vb = sV + static_cast<uint32_t>(bb) * SLOT;
      const bool leader = elect_one();
      for (int kk = 0; kk < prev_keys / 16; ++kk) {
        const uint64_t bd = mnmaj | ((vb + kk * 2048) >> 4);
        if (leader)
          mma_bf16_ts(tmem + O_COL, aP + kk * 8, bd, idesc_pv, (!prev_first || kk > 0) ? 1u : 0u);
      }
      if (leader) {
        mma_commit(smem_u32(&v_empty[bb]));
        mma_commit(smem_u32(&s_free[bb]));
        if (prev_last) mma_commit(smem_u32(&o_full));
      }
      __syncwarp();
      return true;
    };
    for (int i = 0; ok; ++i) {
      int u = -1, P = 0;
      if (!read_unit(i, u, P)) break;
      if (u < 0) break;
      int b, s, g;
      unit_of(u, b, s, g);
      const Range rg = range_of(s, P);
      // Q slots go to the units with steps, in turn
      const int qs = units_o % kSplTcQSlots;
      if (rg.nsteps > 0 && !wait_all(q_full[qs], (units_o / kSplTcQSlots) & 1)) break;
      const uint64_t aq = amaj | ((sQ + qs * NCH * 4096) >> 4);
      for (int k = 0; k < rg.nsteps; ++k, ++n) {
        const int bb = n & 1, ks = n % kSplTcKSlots;
        const bool cached = k < rg.ncached;
        const int keys = cached ? 128 : 16;
        if (!wait_all(s_free[bb], ((n >> 1) & 1) ^ 1) ||
            !wait_all(k_full[ks], (n / kSplTcKSlots) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bk = kmaj | ((sK + ks * SLOT) >> 4);
        const uint32_t idesc_s = idesc_bf16_f32(64, keys, false, false);
        const bool leader = elect_one();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = ((kk >> 2) * 4096 + (kk & 3) * 32) >> 4;
          const uint32_t offk = ((kk >> 2) * 128 * 128 + (kk & 3) * 32) >> 4;
          if (leader)
            mma_bf16_ss(tmem + bb * S_COLS, aq + offq, bk + offk, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          mma_commit(smem_u32(&s_full[bb]));
          mma_commit(smem_u32(&k_empty[ks]));
          if (k == rg.nsteps - 1) mma_commit(smem_u32(&q_empty[qs]));
        }
        __syncwarp();
        if (prev && !issue_pv()) {
          ok = false;
          break;
        }
        prev = true;
        prev_first = k == 0;
        prev_last = k == rg.nsteps - 1;
        prev_keys = keys;
        if (prev_first) prev_o = units_o++;
      }
    }
    if (ok && prev) issue_pv();  // P V of the last step (n - 1)
  } else if (warp == 9) {
    // ======================= TMA producer ====================================
    // Units: this CTA's own, then those of cancelled launches. Per unit: Q,
    // then its steps: K of step n (slot freed by S(n-3)), V of step n - 2.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_vc);
      tma_prefetch_desc(&tm_kn);
      tma_prefetch_desc(&tm_vn);
      auto publish = [&](int j, int u, int P) -> bool {
        const int e = j % kDecTcUnits;
        if (!mbar_wait(smem_u32(&ur_empty[e]), ((j / kDecTcUnits) & 1) ^ 1, abort)) return false;
        ring_u[e] = u;
        ring_P[e] = P;
        mbar_arrive(smem_u32(&ur_full[e]));
        return true;
      };
      // step loads: K or V of one step of unit (b, g, range rg), into slot dst
      // on bar; returns the bytes
      auto step_boxes = [&](const CUtensorMap* tc, const CUtensorMap* tn, uint32_t dst,
                            uint32_t bar, int b, int g, const Range& rg, int k) {
        if (k < rg.ncached) {
          const int tiles = min(2, rg.ntile - 2 * k);
          mbar_arrive_expect_tx(bar, static_cast<uint32_t>(tiles) * NCH * T * 128);
          for (int h = 0; h < tiles; ++h) {
            const int slot = (rg.t0 + (2 * k + h) * T) % W;  // W % T == 0: no wrap
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
              tma_load_4d(dst + ch * 128 * 128 + h * T * 128, tc, bar, ch * 64, g, slot, b);
          }
        } else {
          mbar_arrive_expect_tx(bar, NCH * n_q * 128);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) tma_load_4d(dst + ch * 128 * 128, tn, bar, ch * 64, g, 0, b);
        }
      };
      // V of an earlier step: its unit's coordinates are kept in a small history
      struct Pend { int b, g, k; Range rg; };
      Pend hist[4];
      int nk = 0, nv = 0;
      auto load_v = [&](const Pend& pd) -> bool {
        const int vs = nv & 1;
        if (!mbar_wait(smem_u32(&v_empty[vs]), ((nv >> 1) & 1) ^ 1, abort)) return false;
        step_boxes(&tm_vc, &tm_vn, sV + vs * SLOT, smem_u32(&v_full[vs]), pd.b, pd.g, pd.rg, pd.k);
        ++nv;
        return true;
      };
      uint32_t clc_phase = 0;
      bool clc_pending = false;
      auto ask = [&]() {
        mbar_arrive_expect_tx(smem_u32(&clc_bar), 16u);
        clc_try_cancel(smem_u32(clc_resp), smem_u32(&clc_bar));
        clc_pending = true;
      };
      int u = static_cast<int>(blockIdx.x);
      ask();
      bool ok = true;
      int i = 0;   // ring entries published
      int nq = 0;  // units with steps (Q slot nq % 2)
      for (;;) {
        int P = 0;
        int b = 0, s = 0, g = 0;
        if (u >= 0) {
          unit_of(u, b, s, g);
          P = __ldg(p.pos + b);
          if (P < 0) {
            if (s == 0) flag_error(2u);
            P = 0;
          }
          const int lo0 = max(0, P - W + 1);
          if (s == p.S - 1 && min(lo0 + (s + 1) * p.chunk, P) < P) flag_error(2u);
        }
        const Range rg = range_of(s, P);
        if (u >= 0 && rg.nsteps == 0) {
          // an empty state: m = -inf for the unit's rows (the merge skips it)
          const int unit = (b * p.Hkv + g) * p.S + s;
          for (int row = 0; row < 32; ++row)
            p.part[(static_cast<size_t>(unit) * 32 + row) * (D + 4) + D] = -INFINITY;
        } else {
          if (!publish(i, u, P)) {
            ok = false;
            break;
          }
          ++i;
          if (u < 0) break;
        }
        if (rg.nsteps > 0) {
          const int qs = nq % kSplTcQSlots;
          if (!mbar_wait(smem_u32(&q_empty[qs]), ((nq / kSplTcQSlots) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          ++nq;
          mbar_arrive_expect_tx(smem_u32(&q_full[qs]), NCH * R * 128);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch)
            tma_load_4d(sQ + (qs * NCH + ch) * 4096, &tm_q, smem_u32(&q_full[qs]), ch * 64,
                        g * G, 0, b);
        }
        for (int k = 0; k < rg.nsteps && ok; ++k) {
          const int ks = nk % kSplTcKSlots;
          if (!mbar_wait(smem_u32(&k_empty[ks]), ((nk / kSplTcKSlots) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          step_boxes(&tm_kc, &tm_kn, sK + ks * SLOT, smem_u32(&k_full[ks]), b, g, rg, k);
          hist[nk & 3] = Pend{b, g, k, rg};
          ++nk;
          if (nk - 2 > nv && !load_v(hist[(nk - 3) & 3])) ok = false;
        }
        if (!ok) break;
        if (!mbar_wait(smem_u32(&clc_bar), clc_phase, abort)) {
          ok = false;
          break;
        }
        clc_phase ^= 1u;
        clc_pending = false;
        int x = -1;
        u = clc_query(smem_u32(clc_resp), x) ? x : -1;
        if (u >= 0) ask();
      }
      while (ok && nv < nk) ok = load_v(hist[nv & 3]);
      // every load has landed before the CTA leaves (bounded on its own)
      int no_abort = 0;
      for (int s2 = 0; s2 < kSplTcKSlots; ++s2) {
        const int last = nk - 1 - ((nk - 1 - s2) % kSplTcKSlots + kSplTcKSlots) % kSplTcKSlots;
        if (last >= 0) mbar_wait(smem_u32(&k_full[s2]), (last / kSplTcKSlots) & 1, &no_abort);
      }
      for (int s2 = 0; s2 < kSplTcVSlots; ++s2) {
        const int last = nv - 1 - ((nv - 1 - s2) % kSplTcVSlots + kSplTcVSlots) % kSplTcVSlots;
        if (last >= 0) mbar_wait(smem_u32(&v_full[s2]), (last >> 1) & 1, &no_abort);
      }
      if (clc_pending) mbar_wait(smem_u32(&clc_bar), clc_phase, &no_abort);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace swa
