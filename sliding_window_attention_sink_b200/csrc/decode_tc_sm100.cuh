// decode_tc_sm100.cuh -- decode / draft verification over a W-slot bf16 KV
// ring on the tcgen05 tensor cores: a persistent kernel, one CTA per SM.
//
// Operation: the same as decode_sm100_kernel (decode_sm100.cuh): n_q new
// tokens per sequence (one real token plus MTP drafts, "MiMo-V2-Flash
// Technical Report" summary, section 2.3) attend to the committed tokens of
// the window in the ring and to the new tokens up to themselves, with the
// per-head sink in the softmax denominator (section 2.2.2).
//
// Design (sm_100a). A unit is one (sequence, kv head): R = n_q * G <= 32
// query rows against KP key rows (the W ring rows, the n_q new rows from row
// W8 = roundup8(W), padding to a multiple of 16).
// * S = Q K^T with the queries on the MMA's M side (M = 64, N = KP, K = D).
//   An M = 64 accumulator puts rows 16q .. 16q+15 in tensor-memory lanes
//   32q .. 32q+15. The A descriptor steps 512 bytes per 8-row group instead
//   of 1024, so that M-row groups 0, 2, 4, 6 read Q rows 0-7, 8-15, 16-23,
//   24-31 (each 1024 bytes into the 128-byte-swizzled slot, where the swizzle
//   phase is the row's own) and land in lanes 32q .. 32q+7: every lane
//   quarter, and so every SM sub-partition, holds 8 real rows. The odd groups
//   read shifted bytes of the same slots; their lanes are never read.
// * Four softmax warps per unit (one per lane quarter) read S with the
//   16-lane x 256-bit shape: 4 threads per row, 2 adjacent keys per thread
//   per 8 keys, row max and sums by quad shuffles. P = exp2(S - m) goes back
//   over S as bf16 pairs with the 16-lane x 128-bit shape, whose column per
//   thread is exactly the pair the thread holds, and O = P V reads it from
//   tensor memory (A from TMEM, V as the MN-major B operand).
// * The grid has one CTA per unit, and one CTA fits an SM. A CTA starts with
//   its own unit and then takes the units of CTAs that have not started,
//   cancelling their launch (cluster launch control), so that the SMs that
//   run ahead do more units and all finish together; the producer warp asks,
//   and hands the units to the other warps through a ring in shared memory.
//   Three Q+K slots and two V slots: K of two units ahead and V of one unit
//   ahead are in flight while a unit is computed (up to 180 KB per SM).
// * Warps: 0-3 and 4-7 the softmax of even and odd units (S buffers 0 and
//   1), 8-11 the epilogue (O / l -> bf16 -> staging -> TMA store), 12 the MMA
//   issuer and TMEM owner, 13 the TMA producer. Registers are granted to the
//   14 warps as to 16, so 128 per thread: a launch at 144 fails.
// Every wait is bounded (mbar_wait); a wait that gives up sets the abort flag
// and the device error bit, every role leaves its loop, and the producer
// waits (bounded again) for the loads it still has in flight.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kDecTcWarps = 14;
constexpr int kDecTcThreads = kDecTcWarps * 32;
constexpr int kDecTcMaxKP = 144;  // key rows the softmax registers hold
constexpr int kDecTcKSlots = 3;   // Q + K slots
constexpr int kDecTcVSlots = 2;   // V slots (also the S buffers, softmax warp groups)
constexpr int kDecTcUnits = 16;   // entries of the unit ring
// readers of a unit-ring entry: the MMA warp, the unit's 4 softmax warps and
// the 4 epilogue warps
constexpr int kDecTcUnitReaders = 9;

struct DecodeTcParams {
  DecodeParams d;       // KP: roundup16(W8 + n_q) <= kDecTcMaxKP
  uint32_t s_stride;    // TMEM columns between the two S buffers
  uint32_t o_col;       // TMEM column of O
  uint32_t tmem_cols;   // columns allocated (a power of two >= 32)
};

// Dynamic shared memory: the three Q slots ([D/64][32 rows][128 bytes]), the
// three K slots and the two V slots ([D/64][KP rows][128 bytes], 128-byte
// swizzle), two O staging tiles ([D/64][32][128]), plus 1 KB to align the
// base. The S MMA's A operand reads up to 4608 bytes from a Q chunk's start,
// past the last Q slot into the K slots.
__host__ __device__ inline size_t decode_tc_smem_bytes(int D, int KP) {
  const size_t nch = static_cast<size_t>(D / 64);
  return 1024 + nch * (kDecTcKSlots * 4096 + kDecTcKSlots * static_cast<size_t>(KP) * 128 +
                       kDecTcVSlots * static_cast<size_t>(KP) * 128 + 2 * 4096);
}

template <int D>
__global__ void __launch_bounds__(kDecTcThreads, 1)
    decode_tc_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_kr,
                           const __grid_constant__ CUtensorMap tm_kn,
                           const __grid_constant__ CUtensorMap tm_vr,
                           const __grid_constant__ CUtensorMap tm_vn,
                           const __grid_constant__ CUtensorMap tm_o, const DecodeTcParams tp) {
  constexpr int NCH = D / 64;
  constexpr int NREP = kDecTcMaxKP / 8;  // 8-key blocks of a row
  const DecodeParams& p = tp.d;
  extern __shared__ uint8_t dtc_smem[];
  __shared__ __align__(8) uint64_t kq_full[kDecTcKSlots], kq_empty[kDecTcKSlots];
  __shared__ __align__(8) uint64_t v_full[kDecTcVSlots], v_empty[kDecTcVSlots];
  __shared__ __align__(8) uint64_t s_full[2], s_free[2], p_full[2], l_free[2];
  __shared__ __align__(8) uint64_t o_full, o_empty;
  __shared__ __align__(8) uint64_t ur_full[kDecTcUnits], ur_empty[kDecTcUnits];
  __shared__ int unit_ring[kDecTcUnits];  // unit ids; -1 after the last
  __shared__ __align__(16) uint32_t clc_resp[4];
  __shared__ __align__(8) uint64_t clc_bar;
  __shared__ float l_s[2][32];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KP = p.KP, W = p.W, W8 = p.W8, n_q = p.n_q, G = p.G, R = p.R;
  const uint32_t slot_kv = static_cast<uint32_t>(NCH * KP * 128);  // one K or V slot
  const uint32_t base = (smem_u32(dtc_smem) + 1023u) & ~1023u;
  const uint32_t sQ = base;                                // 3 x NCH x 4096
  const uint32_t sK = sQ + kDecTcKSlots * NCH * 4096;      // 3 x slot_kv
  const uint32_t sV = sK + kDecTcKSlots * slot_kv;         // 2 x slot_kv
  const uint32_t sO = sV + kDecTcVSlots * slot_kv;         // 2 x NCH x 4096

  if (tid == 0) {
    for (int s = 0; s < kDecTcKSlots; ++s) {
      mbar_init(smem_u32(&kq_full[s]), 1);
      mbar_init(smem_u32(&kq_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_free[s]), 1);
      mbar_init(smem_u32(&p_full[s]), 4);
      mbar_init(smem_u32(&l_free[s]), 4);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), 4);
    for (int s = 0; s < kDecTcUnits; ++s) {
      mbar_init(smem_u32(&ur_full[s]), 1);
      mbar_init(smem_u32(&ur_empty[s]), kDecTcUnitReaders);
    }
    mbar_init(smem_u32(&clc_bar), 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_u32(&tmem_base_sh), tp.tmem_cols);
    tmem_relinquish();
  }
  // V rows that no box writes (between the ring and the new rows, and after
  // the new rows) are zero in both V slots for the whole launch: P is 0
  // there, and 0 * V must stay 0
  {
    const int pad1 = W8 - W, pad2 = KP - (W8 + n_q);
    const int per_slot = NCH * (pad1 + pad2) * 8;  // 16-byte units
    for (int idx = tid; idx < kDecTcVSlots * per_slot; idx += kDecTcThreads) {
      const int vs = idx / per_slot;
      const int rem0 = idx - vs * per_slot;
      const int ch = rem0 / ((pad1 + pad2) * 8);
      const int rem = rem0 - ch * (pad1 + pad2) * 8;
      const int pr = rem >> 3;
      const int row = pr < pad1 ? W + pr : W8 + n_q + (pr - pad1);
      st_shared_zero16(sV + vs * slot_kv + ch * KP * 128 + row * 128 + (rem & 7) * 16);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // a wait taken by a whole warp: every lane gets the same answer, so the
  // warp leaves its loop together
  auto wait_all = [&](uint64_t& bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar), parity, abort));
  };
  auto unit_of = [&](int u, int& bs, int& g) {
    bs = u / p.Hkv;
    g = u - bs * p.Hkv;
  };
  // the i-th unit of this CTA (-1: none left), read by a whole warp, which
  // then releases the entry; false when the wait gave up
  auto read_unit = [&](int i, int& u) -> bool {
    const int e = i % kDecTcUnits;
    if (!wait_all(ur_full[e], (i / kDecTcUnits) & 1)) return false;
    u = unit_ring[e];
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ur_empty[e]));
    return true;
  };

  if (warp < 8) {
    // ================== softmax (4 warps per unit, 8 rows each) ==============
    const int q4 = warp & 3;   // lane quarter
    const int grp = warp >> 2;  // units i = grp, grp + 2, ...; S buffer grp
    const int s4 = lane & 3;   // this thread's keys: 8k + 2*s4 and + 1
    const int r = 8 * q4 + (lane >> 2);  // query row (TMEM lane 32*q4 + lane/4)
    const bool rvalid = r < R;
    const int t = rvalid ? r / G : -1;
    const int hh = rvalid ? r - t * G : 0;
    const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
    const uint32_t tS = tmem + (static_cast<uint32_t>(32 * q4) << 16) +
                        static_cast<uint32_t>(grp) * tp.s_stride;
    // the position and sink of this warp's next unit, loaded a unit ahead
    // (a global load's latency under a full memory system is microseconds)
    auto fetch = [&](int u, int& P, float& sk) {
      if (u >= 0) {
        int bs, g;
        unit_of(u, bs, g);
        P = __ldg(p.pos + bs);
        sk = (rvalid && p.sink != nullptr) ? __ldg(p.sink + g * G + hh) : -INFINITY;
      }
    };
    int u_next = -1;
    int P_next = 0;
    float sk_next = -INFINITY;
    if (read_unit(grp, u_next)) fetch(u_next, P_next, sk_next);
    for (int i = grp; u_next >= 0; i += 2) {
      const int u = u_next;
      int bs, g;
      unit_of(u, bs, g);
      int P = P_next;
      const float sink2 = sk_next * kLog2e;
      // (the ring ends with two -1 entries, one for each warp group)
      if (!read_unit(i + 2, u_next)) break;
      fetch(u_next, P_next, sk_next);
      if (P < 0) {
        if (lane == 0 && q4 == 0) flag_error(2u);
        P = 0;
      }
      // Key ranks: ring slot s holds the token at position P - W + rel(s),
      // rel(s) = (s - P) mod W; new token u has rank W + u. Query t sees ring
      // ranks >= lo = max(t + 1, W - P) and new tokens u <= t. The columns it
      // does not see: the cyclic run of L = min(lo, W) ring slots from P mod W,
      // the padding [W, W8), and from new row t + 1 on (an invalid row, t = -1,
      // sees nothing). As bit masks over this thread's 8-key blocks k, one per
      // key 8k + 2*s4 + e, so that masking takes no branch.
      uint32_t inv[2];
      {
        const int Pmod = P % W;
        const int L = rvalid ? min(max(t + 1, W - P), W) : W;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          // blocks k whose key 8k + 2*s4 + e lies in [x0, x1)
          auto blocks = [&](int x0, int x1) -> uint32_t {
            const int k0 = min(NREP, max(0, (x0 - 2 * s4 - e + 7) >> 3));
            const int k1 = min(NREP, max(0, (x1 - 2 * s4 - e + 7) >> 3));
            return k1 > k0 ? (1u << k1) - (1u << k0) : 0u;
          };
          inv[e] = blocks(Pmod, min(Pmod + L, W)) | blocks(0, Pmod + L - W) | blocks(W, W8) |
                   blocks(W8 + t + 1, 8 * NREP);
        }
      }
      if (!wait_all(s_full[grp], (i >> 1) & 1)) break;
      tc_fence_after();
      // S: 8-key block k in v[4k], v[4k+1] (v[4k+2], v[4k+3]: lane 8 + row)
      uint32_t v[NREP * 4];
#pragma unroll
      for (int m = 0; m < NREP / 4; ++m) {
        if (32 * m + 32 <= KP) tmem_ld_16x256b_x4(tS + 32 * m, &v[16 * m]);
        else if (32 * m + 16 <= KP) tmem_ld_16x256b_x2(tS + 32 * m, &v[16 * m]);
      }
      if constexpr (NREP % 4 != 0) {
        constexpr int m = NREP / 4;
        if (32 * m + 16 <= KP) tmem_ld_16x256b_x2(tS + 32 * m, &v[16 * m]);
      }
      tmem_ld_wait();
      // (blocks past KP were not loaded: they are in the mask)
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < NREP; ++k) {
        v[4 * k] = ((inv[0] >> k) & 1u) ? 0xff800000u : v[4 * k];
        v[4 * k + 1] = ((inv[1] >> k) & 1u) ? 0xff800000u : v[4 * k + 1];
        mx = max3(mx, __uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]));
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m = fmaxf(sink2, mx * p.scale_log2);
      const float mb = (m == -INFINITY) ? 0.f : m;
      // P = exp2(x - m) (masked: exp2(-inf) = 0) as bf16 pairs over S: the
      // pair of keys 8k + 2*s4, + 1 is P column 4k + s4 (lane 8 + row gets a
      // copy: a row nobody reads). Sums of the rounded P (for O) and of fp32 P
      // (for the LSE).
      uint64_t lr2 = 0, lx2 = 0;
      const uint64_t nm2 = f2_pack(-mb, -mb);
      uint32_t w[NREP];
#pragma unroll
      for (int k = 0; k < NREP; ++k) {
        float t0f, t1f;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1])), sc2,
                         nm2),
                  t0f, t1f);
        const float x0 = ex2(t0f), x1 = ex2(t1f);
        const uint32_t pk = pack_bf16x2(x0, x1);
        w[k] = pk;
        lr2 = f2_add(lr2, f2_pack(bf16lo_to_f32(pk), bf16hi_to_f32(pk)));
        lx2 = f2_add(lx2, f2_pack(x0, x1));
      }
#pragma unroll
      for (int m = 0; m < NREP / 8; ++m) {
        // P columns [32m, 32m + 32) hold the keys [64m, 64m + 64)
        if (64 * m + 64 <= KP) {
          tmem_st_16x128b_x8_dup(tS + 32 * m, &w[8 * m]);
        } else {
          // 0, 16, 32 or 48 keys left: blocks of 16 keys (8 P columns)
#pragma unroll
          for (int h = 0; h < 3; ++h)
            if (64 * m + 16 * h + 16 <= KP)
              tmem_st_16x128b_x2_dup(tS + 32 * m + 8 * h, &w[8 * m + 2 * h]);
        }
      }
#pragma unroll
      for (int h = 0; h < (NREP % 8) / 2; ++h) {
        constexpr int m = NREP / 8;
        if (64 * m + 16 * h + 16 <= KP) tmem_st_16x128b_x2_dup(tS + 32 * m + 8 * h, &w[8 * m + 2 * h]);
      }
      float l_r, l_x;
      {
        float a0, a1;
        f2_unpack(lr2, a0, a1);
        l_r = a0 + a1;
        f2_unpack(lx2, a0, a1);
        l_x = a0 + a1;
      }
      l_r += __shfl_xor_sync(0xffffffffu, l_r, 1);
      l_x += __shfl_xor_sync(0xffffffffu, l_x, 1);
      l_r += __shfl_xor_sync(0xffffffffu, l_r, 2);
      l_x += __shfl_xor_sync(0xffffffffu, l_x, 2);
      if (sink2 != -INFINITY) {
        const float ts = ex2(sink2 - mb);
        l_r += ts;
        l_x += ts;
      }
      // with fewer than W committed tokens the slots P .. W-1 were never
      // written and may hold anything: their P is 0, and 0 * V must stay 0
      // (the four warps of the group split the rows' 16-byte units)
      bool ok = true;
      if (P < W) {
        ok = mbar_wait(smem_u32(&v_full[grp]), (i >> 1) & 1, abort);
        if (ok) {
          const uint32_t vslot = sV + static_cast<uint32_t>(grp) * slot_kv;
          for (int idx = q4 * 32 + lane; idx < NCH * (W - P) * 8; idx += 128) {
            const int ch = idx / ((W - P) * 8);
            const int rem = idx - ch * (W - P) * 8;
            st_shared_zero16(vslot + ch * KP * 128 + (P + (rem >> 3)) * 128 + (rem & 7) * 16);
          }
          fence_proxy_async_smem();
        }
      }
      // l for the epilogue, once it has read this buffer's previous value
      if (ok) ok = mbar_wait(smem_u32(&l_free[grp]), ((i >> 1) & 1) ^ 1, abort);
      if (ok && s4 == 0) l_s[grp][r] = l_r;
      tmem_st_wait();
      tc_fence_before();
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0) mbar_arrive(smem_u32(&p_full[grp]));
      if (rvalid && s4 == 0 && p.lse != nullptr)
        p.lse[(static_cast<size_t>(bs) * n_q + t) * p.Hq + g * G + hh] = (mb + lg2(l_x)) * kLn2;
    }
  } else if (warp < 12) {
    // ================== epilogue (4 warps, 8 rows each) ======================
    const int q4 = warp & 3;
    const int s4 = lane & 3;
    const int r = 8 * q4 + (lane >> 2);
    const bool issuer = warp == 8 && lane == 0;
    const uint32_t tO = tmem + (static_cast<uint32_t>(32 * q4) << 16) + tp.o_col;
    for (int i = 0;; ++i) {
      const int b = i & 1;
      int u = -1;
      const bool got = read_unit(i, u);
      if (named_bar_any(1, 128, !got || u < 0)) break;  // the four warps leave together
      int bs, g;
      unit_of(u, bs, g);
      // p_full of the unit completed before its PV was issued; waiting on it
      // too orders the softmax's write of l_s[b] before the read below
      const bool ok = wait_all(o_full, i & 1) && wait_all(p_full[b], (i >> 1) & 1);
      if (named_bar_any(1, 128, !ok)) break;
      tc_fence_after();
      const float l = l_s[b][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&l_free[b]));
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      uint32_t o[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_16x256b_x4(tO + 32 * c, &o[16 * c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&o_empty));
      // this unit's staging tile is free once the store of unit i-2 has read it
      if (issuer) tma_store_wait_read<1>();
      named_bar_sync(1, 128);
      const uint32_t stg = sO + static_cast<uint32_t>(b) * NCH * 4096;
#pragma unroll
      for (int k = 0; k < D / 8; ++k) {
        // columns 8k + 2*s4, + 1: 16-byte unit k % 8 of chunk k / 8, bytes 4*s4
        const uint32_t a = stg + (k >> 3) * 4096 + r * 128 + ((((k & 7) ^ (r & 7))) << 4) + 4 * s4;
        const uint32_t pk = pack_bf16x2(__uint_as_float(o[4 * k]) * inv_l,
                                        __uint_as_float(o[4 * k + 1]) * inv_l);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(pk) : "memory");
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (issuer) {
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) tma_store_4d(&tm_o, stg + ch * 4096, ch * 64, g * G, 0, bs);
        tma_store_commit();
      }
    }
    if (issuer) tma_store_wait_all<0>();
  } else if (warp == 12) {
    // ======================= MMA issuer ======================================
    // S(i) = Q K^T, then O(i-1) = P V: S of the next unit is on the tensor
    // cores while the softmax of this one runs.
    const uint64_t amaj = smem_desc_sw128(0, 16, 512);   // Q: 8-row groups 512 B apart
    const uint64_t kmaj = smem_desc_sw128(0, 16, 1024);  // K: K-major
    const uint64_t mnmaj = smem_desc_sw128(0, NCH > 1 ? KP * 128 : 16, 1024);  // V: MN-major
    const uint32_t idesc_s = idesc_bf16_f32(64, KP, false, false);
    const uint32_t idesc_pv = idesc_bf16_f32(64, D, false, true);
    for (int i = 0;; ++i) {
      int u = -1;
      if (!read_unit(i, u)) break;
      const bool has = u >= 0;  // unit i exists
      if (has) {
        const int b = i & 1, ks = i % kDecTcKSlots;
        if (!wait_all(s_free[b], ((i >> 1) & 1) ^ 1)) break;
        if (!wait_all(kq_full[ks], (i / kDecTcKSlots) & 1)) break;
        tc_fence_after();
        const uint64_t aq = amaj | ((sQ + ks * NCH * 4096) >> 4);
        const uint64_t bk = kmaj | ((sK + ks * slot_kv) >> 4);
        const bool leader = elect_one();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = ((kk >> 2) * 4096 + (kk & 3) * 32) >> 4;
          const uint32_t offk = ((kk >> 2) * KP * 128 + (kk & 3) * 32) >> 4;
          if (leader)
            mma_bf16_ss(tmem + b * tp.s_stride, aq + offq, bk + offk, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          mma_commit(smem_u32(&s_full[b]));
          mma_commit(smem_u32(&kq_empty[ks]));
        }
        __syncwarp();
      }
      if (i >= 1) {
        const int j = i - 1, b = j & 1;
        if (!wait_all(p_full[b], (j >> 1) & 1)) break;
        if (!wait_all(v_full[b], (j >> 1) & 1)) break;
        if (!wait_all(o_empty, (j & 1) ^ 1)) break;
        tc_fence_after();
        const uint32_t aP = tmem + b * tp.s_stride;  // P: 8 columns per 16 keys
        const uint32_t vb = sV + b * slot_kv;
        const bool leader = elect_one();
        for (int kk = 0; kk < KP / 16; ++kk) {
          const uint64_t bd = mnmaj | ((vb + kk * 2048) >> 4);
          if (leader) mma_bf16_ts(tmem + tp.o_col, aP + kk * 8, bd, idesc_pv, kk > 0 ? 1u : 0u);
        }
        if (leader) {
          mma_commit(smem_u32(&o_full));
          mma_commit(smem_u32(&v_empty[b]));
          mma_commit(smem_u32(&s_free[b]));
        }
        __syncwarp();
      }
      if (!has) break;
    }
  } else {
    // ======================= TMA producer (warp 13) ==========================
    // Units: this CTA's own, then those of cancelled launches, published in
    // the unit ring (two -1 entries after the last). Loads in the order their
    // slots come free: Q+K of unit j (slot freed by S(j-3)), then V of unit
    // j-2 (freed by O(j-4)). The next unit is asked for while this one's
    // loads are issued.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kr);
      tma_prefetch_desc(&tm_kn);
      tma_prefetch_desc(&tm_vr);
      tma_prefetch_desc(&tm_vn);
      const uint32_t kv_bytes = NCH * (W + n_q) * 128;
      auto publish = [&](int j, int u) -> bool {
        const int e = j % kDecTcUnits;
        if (!mbar_wait(smem_u32(&ur_empty[e]), ((j / kDecTcUnits) & 1) ^ 1, abort)) return false;
        unit_ring[e] = u;
        mbar_arrive(smem_u32(&ur_full[e]));
        return true;
      };
      auto load_v = [&](int jv, int u) -> bool {
        const int vs = jv & 1;
        if (!mbar_wait(smem_u32(&v_empty[vs]), ((jv >> 1) & 1) ^ 1, abort)) return false;
        int bs, g;
        unit_of(u, bs, g);
        const uint32_t bar = smem_u32(&v_full[vs]);
        mbar_arrive_expect_tx(bar, kv_bytes);
        const uint32_t vd = sV + vs * slot_kv;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) {
          tma_load_4d(vd + ch * KP * 128, &tm_vr, bar, ch * 64, g, 0, bs);
          tma_load_4d(vd + ch * KP * 128 + W8 * 128, &tm_vn, bar, ch * 64, g, 0, bs);
        }
        return true;
      };
      int nk = 0, nv = 0;         // loads issued
      int hist[2] = {-1, -1};     // units j-1 and j-2
      uint32_t clc_phase = 0;
      bool clc_pending = false;   // a cancellation request is in flight
      int u = static_cast<int>(blockIdx.x);
      auto ask = [&]() {
        mbar_arrive_expect_tx(smem_u32(&clc_bar), 16u);
        clc_try_cancel(smem_u32(clc_resp), smem_u32(&clc_bar));
        clc_pending = true;
      };
      ask();
      bool ok = true;
      int j = 0;
      for (;; ++j) {
        if (!publish(j, u)) {
          ok = false;
          break;
        }
        if (u < 0) break;
        const int ks = j % kDecTcKSlots;
        if (!mbar_wait(smem_u32(&kq_empty[ks]), ((j / kDecTcKSlots) & 1) ^ 1, abort)) {
          ok = false;
          break;
        }
        {
          int bs, g;
          unit_of(u, bs, g);
          const uint32_t bar = smem_u32(&kq_full[ks]);
          mbar_arrive_expect_tx(bar, NCH * R * 128 + kv_bytes);
          const uint32_t qd = sQ + ks * NCH * 4096, kd = sK + ks * slot_kv;
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            tma_load_4d(qd + ch * 4096, &tm_q, bar, ch * 64, g * G, 0, bs);
            tma_load_4d(kd + ch * KP * 128, &tm_kr, bar, ch * 64, g, 0, bs);
            tma_load_4d(kd + ch * KP * 128 + W8 * 128, &tm_kn, bar, ch * 64, g, 0, bs);
          }
          ++nk;
        }
        if (j >= 2) {
          if (!load_v(j - 2, hist[1])) {
            ok = false;
            break;
          }
          ++nv;
        }
        hist[1] = hist[0];
        hist[0] = u;
        // the next unit: a cancelled launch's, or none
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
      // j: the number of units; the second -1 entry, and the last V loads
      if (ok) ok = publish(j + 1, -1);
      for (int jv = max(j - 2, 0); ok && jv < j; ++jv) {
        ok = load_v(jv, jv == j - 1 ? hist[0] : hist[1]);
        if (ok) ++nv;
      }
      // Each slot has at most one load in flight (its previous one was
      // consumed before the slot was refilled): wait for the last load of
      // every slot, and for a cancellation response still in flight, so
      // that nothing lands after the CTA has left. Already complete on the
      // normal path; bounded on its own after an abort.
      int no_abort = 0;
      for (int s2 = 0; s2 < kDecTcKSlots; ++s2) {
        const int last = nk - 1 - ((nk - 1 - s2) % kDecTcKSlots + kDecTcKSlots) % kDecTcKSlots;
        if (last >= 0) mbar_wait(smem_u32(&kq_full[s2]), (last / kDecTcKSlots) & 1, &no_abort);
      }
      for (int s2 = 0; s2 < kDecTcVSlots; ++s2) {
        const int last = nv - 1 - ((nv - 1 - s2) % kDecTcVSlots + kDecTcVSlots) % kDecTcVSlots;
        if (last >= 0) mbar_wait(smem_u32(&v_full[s2]), (last >> 1) & 1, &no_abort);
      }
      if (clc_pending) mbar_wait(smem_u32(&clc_bar), clc_phase, &no_abort);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, tp.tmem_cols);
  }
}

}  // namespace swa
