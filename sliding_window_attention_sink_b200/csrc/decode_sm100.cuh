// decode_sm100.cuh -- decode / draft verification over a W-slot KV ring, and
// the commit of accepted tokens into the ring.
//
// Operation: the same sink attention as the prefill ("MiMo-V2-Flash Technical
// Report" summary, mlpod.com, section 2.2.2), for n_q new tokens per sequence:
// one real token plus the drafts of the MTP layers, verified in parallel
// (section 2.3 "Lightweight MTP": verification raises arithmetic intensity
// without adding KV-cache I/O). New token t at absolute position P + t sees
// the committed tokens at positions >= P + t - W + 1 (slot p mod W of the
// ring) and the new tokens 0..t.
//
// Design (sm_100a): one CTA per (sequence, kv head); split-free. 4 warps and
// one buffer for K then V when the keys fit (KP <= 160: five CTAs share an
// SM for a 128-slot ring), else 8 warps and separate K and V buffers.
// * All G query heads of the kv head and all n_q tokens are one set of
//   R = n_q * G query rows (32 for n_q = 4, G = 8), so each ring byte is read
//   from HBM exactly once for all of them.
// * One thread issues all loads as TMA boxes into shared memory (128-byte
//   swizzle, 64 head-dim columns per box): the ring slice (W rows of D bf16,
//   Hkv * D apart in HBM) and the n_q new rows of K, then of V, plus the Q
//   rows; K and Q complete on one mbarrier, V on a second one that lands
//   while the scores are computed (with one buffer: V is loaded over K once
//   S is done, while the softmax runs). (16-byte cp.async from every thread took
//   about a third of a CTA's cycles just to issue.) The new rows go to row
//   roundup8(W) so that every box starts on a 1024-byte swizzle atom.
// * The contraction has ~25 flop per HBM byte, above what CUDA-core FMAs hide,
//   so S = Q K^T and O = P V use the tensor cores, here through mma.sync m16n8k16
//   (bf16, f32 accumulate); rings of <= 144 padded keys take decode_tc_sm100.cuh.
//   ldmatrix addresses follow the swizzle.
// * Softmax: the warps split the keys for S; row maxima and sums are
//   reduced inside the quad that shares a row (warp shuffles), then across
//   warps through shared memory. The max is seeded with the sink logit and
//   the denominator gets the sink term exp(s - m). P goes to shared memory as
//   bf16 over Q's place; the warps then split the head dim for O = P V.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx_sm100.cuh"

namespace swa {

struct DecodeParams {
  const __nv_bfloat16 *q, *k_new, *v_new, *k_ring, *v_ring;
  const int32_t* pos;
  int B, n_q, Hq, Hkv, G, W;
  int R;    // query rows per CTA = n_q * G (<= 32)
  int W8;   // first row of the new keys: roundup8(W)
  int KP;   // key rows padded to a multiple of 16: roundup16(W8 + n_q)
  const float* sink;
  float scale_log2;
  __nv_bfloat16* o;
  float* lse;
};

__device__ __forceinline__ void st_shared_zero16(uint32_t dst) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                        uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x1_t(uint32_t addr, uint32_t& r0) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x1.trans.shared.b16 {%0}, [%1];"
               : "=r"(r0)
               : "r"(addr));
}

// D += A B on m16n8k8 (bf16 in, f32 accumulate): the last 8 keys of PV.
__device__ __forceinline__ void mma_1688(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                          uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

// Warps per CTA: 4 when the keys fit 5 n8 tiles per warp (KP <= 160), with
// one shared-memory buffer that holds K and then V, so that four CTAs share
// an SM and overlap their loads; else 8 warps with separate K and V buffers.
constexpr int kDecodeSmallWarps = 4;
constexpr int kDecodeLargeWarps = 8;
constexpr int kDecodeSmallMaxKP = 160;

// Shared memory (the dynamic region, 1024-byte aligned; no static shared
// memory): K and V (or one buffer for both) as D/64 blocks of [KP rows][128
// bytes]; Q as D/64 blocks of [32 rows][128 bytes] (128-byte swizzle: 16-byte
// unit u of row r at u ^ (r & 7)), later overwritten by P [32][LDP] bf16;
// then per-warp row maxima and the two row sums [NWP][32], per-row l [32]
// (fp32), and the two mbarriers and the abort flag. KP is a multiple of 8;
// P rows are KP + 8 apart when KP is a multiple of 16 (a 16-byte shift per
// row keeps ldmatrix free of bank conflicts), else KP apart (already so).
// With W = 128 and n_q <= 4 the 4-warp CTA takes 45 216 bytes: five share an SM.
__host__ __device__ inline int decode_ldp(int KP) { return (KP % 16 == 8) ? KP : KP + 8; }
__host__ __device__ inline size_t decode_qp_bytes(int D, int KP) {
  const size_t q = static_cast<size_t>(D / 64) * 32 * 128;
  const size_t pb = static_cast<size_t>(32) * decode_ldp(KP) * 2;
  return q > pb ? q : pb;
}
__host__ __device__ inline size_t decode_smem_bytes(int D, int KP, int nwp) {
  const size_t kv = static_cast<size_t>(D / 64) * KP * 128 * (nwp == kDecodeSmallWarps ? 1 : 2);
  return kv + decode_qp_bytes(D, KP) + (static_cast<size_t>(nwp) * 32 * 3 + 32) * sizeof(float) +
         32;
}

// Byte address of (row, col) in a tile stored as 64-column blocks of `rows`
// 128-byte rows with the 128-byte swizzle; col a multiple of 8.
__device__ __forceinline__ uint32_t sw128_addr(uint32_t base, int rows, int row, int col) {
  return base + static_cast<uint32_t>((col >> 6) * rows * 128 + row * 128 +
                                      ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

template <int D, int MT, int NWP>
__global__ void __launch_bounds__(NWP * 32, NWP == kDecodeSmallWarps ? 5 : 2)
    decode_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_kr,
                        const __grid_constant__ CUtensorMap tm_kn,
                        const __grid_constant__ CUtensorMap tm_vr,
                        const __grid_constant__ CUtensorMap tm_vn,
                        const __grid_constant__ CUtensorMap tm_o, const DecodeParams p) {
  constexpr bool SHARE = NWP == kDecodeSmallWarps;  // one buffer for K, then V
  constexpr int NT_ = NWP * 32;
  constexpr int NCH = D / 64;      // 64-column blocks of the head dim
  constexpr int RP = MT * 16;      // padded query rows
  constexpr int NTW = 5;           // max n8 key tiles per warp (KP <= 40 * NWP)
  constexpr int DW = D / NWP;      // PV: head-dim columns per warp
  constexpr int NTO = DW / 8;      // n8 tiles per warp in PV (1, 2 or 4)
  extern __shared__ __align__(1024) uint8_t decode_smem[];
  uint8_t* smem_raw = decode_smem;
  const int KP = p.KP;
  const uint32_t sK = smem_u32(smem_raw);
  const uint32_t sV = SHARE ? sK : sK + NCH * KP * 128;
  const uint32_t sQ = sV + NCH * KP * 128;
  // P takes Q's place once S is done
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(smem_raw + (sQ - sK));
  const int LDP = decode_ldp(KP);
  float* red_max = reinterpret_cast<float*>(smem_raw + (sQ - sK) +
                                              decode_qp_bytes(D, KP));  // [NWP][32]
  float* red_lr = red_max + NWP * 32;                         // [NWP][32]
  float* red_lx = red_lr + NWP * 32;                          // [NWP][32]
  float* row_l = red_lx + NWP * 32;                           // [32]
  uint64_t& bar_qk = *reinterpret_cast<uint64_t*>(row_l + 32);
  uint64_t& bar_v = *(&bar_qk + 1);
  int& abort_sh = *reinterpret_cast<int*>(&bar_qk + 2);
  volatile int* abort = &abort_sh;
  // the swizzled TMA boxes need a 1024-byte aligned base (the region starts
  // there when the kernel has no static shared memory)
  if (sK & 1023u) {
    if (threadIdx.x == 0) flag_error(2u);
    return;
  }

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / p.Hkv;
  const int g = blockIdx.x - b * p.Hkv;
  const int W = p.W, n_q = p.n_q, G = p.G;

  // ---- loads: Q and K on bar_qk, V on bar_v (one thread issues) ------------
  const int W8 = p.W8;
  if (tid == 0) {
    mbar_init(smem_u32(&bar_qk), 1);
    mbar_init(smem_u32(&bar_v), 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kr);
    tma_prefetch_desc(&tm_kn);
    tma_prefetch_desc(&tm_vr);
    tma_prefetch_desc(&tm_vn);
    const uint32_t kv_bytes = NCH * (W + n_q) * 128;
    mbar_arrive_expect_tx(smem_u32(&bar_qk), NCH * p.R * 128 + kv_bytes);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      tma_load_4d(sQ + ch * 32 * 128, &tm_q, smem_u32(&bar_qk), ch * 64, g * G, 0, b);
      tma_load_4d(sK + ch * KP * 128, &tm_kr, smem_u32(&bar_qk), ch * 64, g, 0, b);
      tma_load_4d(sK + ch * KP * 128 + W8 * 128, &tm_kn, smem_u32(&bar_qk), ch * 64, g, 0, b);
    }
    if (!SHARE) {
      mbar_arrive_expect_tx(smem_u32(&bar_v), kv_bytes);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        tma_load_4d(sV + ch * KP * 128, &tm_vr, smem_u32(&bar_v), ch * 64, g, 0, b);
        tma_load_4d(sV + ch * KP * 128 + W8 * 128, &tm_vn, smem_u32(&bar_v), ch * 64, g, 0, b);
      }
    }
  }
  // V rows no box writes (between the ring and the new rows, and after the
  // new rows) are zeroed: P is 0 there, and 0 * V must stay 0 (with one
  // buffer, K's boxes leave the same rows alone)
  {
    const int pad1 = W8 - W, pad2 = KP - (W8 + n_q);
    for (int idx = tid; idx < NCH * (pad1 + pad2) * 8; idx += NT_) {
      const int ch = idx / ((pad1 + pad2) * 8);
      const int rem = idx - ch * (pad1 + pad2) * 8;
      const int pr = rem >> 3;
      const int row = pr < pad1 ? W + pr : W8 + n_q + (pr - pad1);
      st_shared_zero16(sV + ch * KP * 128 + row * 128 + (rem & 7) * 16);
    }
  }

  // ---- this thread's rows (fragment rows lane/4 and lane/4 + 8 per m-tile) --
  // (read after the loads are on their way)
  int P = __ldg(p.pos + b);
  if (P < 0) {
    if (tid == 0) flag_error(2u);
    P = 0;
  }
  // Key ranks: ring slot s holds the token at position P - W + rel(s) with
  // rel(s) = (s - P) mod W, rank rel(s); new token u has rank W + u. Query t
  // sees ring tokens with rel >= max(t + 1, W - P) and new tokens u <= t: the
  // ranks [lo_t, W + t], one contiguous range.
  const int Pmod = P % W;
  int trow[MT][2], rlo[MT][2];
  unsigned rspan[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      const int t = row < p.R ? row / G : -1;  // -1: padding row, sees nothing
      trow[mt][hf] = t;
      rlo[mt][hf] = t >= 0 ? max(t + 1, W - P) : 0x7fffffff;
      rspan[mt][hf] = t >= 0 ? static_cast<unsigned>(W + t - rlo[mt][hf]) : 0u;
    }
  // the sinks of this thread's rows (log2 units), fetched while the loads fly
  float srow[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      srow[mt][hf] = (trow[mt][hf] >= 0 && p.sink != nullptr)
                         ? __ldg(p.sink + g * G + (row - trow[mt][hf] * G)) * kLog2e
                         : -INFINITY;
    }
  float sk_tid = -INFINITY;  // the sink of row tid, for the row sums below
  if (tid < p.R && p.sink != nullptr) {
    const int t = tid / G;
    sk_tid = __ldg(p.sink + g * G + (tid - t * G)) * kLog2e;
  }

  // Q and K in shared memory (the zeroing above is published by the same
  // barrier); a wait that gave up ends every thread of the CTA here
  if (!__syncthreads_and(mbar_wait(smem_u32(&bar_qk), 0, abort))) return;

  // ---- S = Q K^T: warp w takes key tiles w, w+8, w+16, ... ----------------
  const int NT = KP / 8;
  float s[MT][NTW][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[mt][j][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int row = mt * 16 + (lane & 15);
      const int col = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(sw128_addr(sQ, 32, row, col), a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
    }
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      const int nt = warp + NWP * j;
      if (nt < NT) {
        uint32_t b0, b1;
        const int key = nt * 8 + (lane & 7);
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x2(sw128_addr(sK, KP, key, col), b0, b1);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          mma_16816(s[mt][j], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
      }
    }
  }

  if (SHARE) {
    // K has been read: V goes into its buffer while the softmax runs
    __syncthreads();
    if (tid == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(smem_u32(&bar_v), NCH * (W + n_q) * 128);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        tma_load_4d(sV + ch * KP * 128, &tm_vr, smem_u32(&bar_v), ch * 64, g, 0, b);
        tma_load_4d(sV + ch * KP * 128 + W8 * 128, &tm_vn, smem_u32(&bar_v), ch * 64, g, 0, b);
      }
    }
  }

  // ---- mask, scale to log2 units, per-warp row max --------------------------
  float mloc[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) mloc[mt][0] = mloc[mt][1] = -INFINITY;
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    const int nt = warp + NWP * j;
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int col = nt * 8 + 2 * (lane & 3) + e2;
      // this key's rank (0x3fffffff: padding, seen by no query)
      int rank = 0x3fffffff;
      if (nt < NT) {
        if (col < W) {
          rank = col - Pmod;
          if (rank < 0) rank += W;
        } else if (col >= W8 && col < W8 + n_q) {
          rank = W + (col - W8);
        }
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const bool vis = static_cast<unsigned>(rank - rlo[mt][hf]) <= rspan[mt][hf];
          float& x = s[mt][j][hf * 2 + e2];
          x = vis ? x * p.scale_log2 : -INFINITY;
          mloc[mt][hf] = fmaxf(mloc[mt][hf], x);
        }
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v = mloc[mt][hf];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
      if ((lane & 3) == 0) red_max[warp * 32 + mt * 16 + (lane >> 2) + hf * 8] = v;
    }
  __syncthreads();

  // ---- row max over warps and the sink; P = exp2(x - m) -> smem; row sums --
  float mrow[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      float m = srow[mt][hf];
#pragma unroll
      for (int w = 0; w < NWP; ++w) m = fmaxf(m, red_max[w * 32 + row]);
      mrow[mt][hf] = (m == -INFINITY) ? 0.f : m;
    }
  float lr[MT][2], lx[MT][2];
  const uint32_t sP = smem_u32(Ps);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    lr[mt][0] = lr[mt][1] = lx[mt][0] = lx[mt][1] = 0.f;
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      const int nt = warp + NWP * j;
      if (nt < NT) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int row = mt * 16 + (lane >> 2) + hf * 8;
          const int col = nt * 8 + 2 * (lane & 3);
          const float p0 = ex2(s[mt][j][2 * hf] - mrow[mt][hf]);
          const float p1 = ex2(s[mt][j][2 * hf + 1] - mrow[mt][hf]);
          const uint32_t pk = pack_bf16x2(p0, p1);
          lr[mt][hf] += bf16lo_to_f32(pk) + bf16hi_to_f32(pk);
          lx[mt][hf] += p0 + p1;
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + (row * LDP + col) * 2), "r"(pk)
                       : "memory");
        }
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v = lr[mt][hf], x = lx[mt][hf];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if ((lane & 3) == 0) {
        red_lr[warp * 32 + mt * 16 + (lane >> 2) + hf * 8] = v;
        red_lx[warp * 32 + mt * 16 + (lane >> 2) + hf * 8] = x;
      }
    }
  // V in shared memory; a wait that gave up ends every thread here
  if (!__syncthreads_and(mbar_wait(smem_u32(&bar_v), 0, abort))) return;
  // with fewer than W committed tokens the slots P .. W-1 were never written
  // and may hold anything: their P is 0, and 0 * V must stay 0
  if (P < W) {
    for (int idx = tid; idx < NCH * (W - P) * 8; idx += NT_) {
      const int ch = idx / ((W - P) * 8);
      const int rem = idx - ch * (W - P) * 8;
      st_shared_zero16(sV + ch * KP * 128 + (P + (rem >> 3)) * 128 + (rem & 7) * 16);
    }
  }
  // row sums over warps plus the sink term; LSE (one thread per row)
  if (tid < RP) {
    const int row = tid;
    const int t = row < p.R ? row / G : -1;
    const float sk = sk_tid;
    float m = sk;
    for (int w = 0; w < NWP; ++w) m = fmaxf(m, red_max[w * 32 + row]);
    const float mb = (m == -INFINITY) ? 0.f : m;
    float l = 0.f, lxs = 0.f;
    for (int w = 0; w < NWP; ++w) {
      l += red_lr[w * 32 + row];
      lxs += red_lx[w * 32 + row];
    }
    if (sk != -INFINITY) {
      const float ts = ex2(sk - mb);
      l += ts;
      lxs += ts;
    }
    row_l[row] = l;
    if (t >= 0 && p.lse != nullptr)
      p.lse[(static_cast<size_t>(b) * n_q + t) * p.Hq + g * G + (row - t * G)] =
          (mb + lg2(lxs)) * kLn2;
  }
  __syncthreads();

  // ---- O = P V: warp w takes head-dim columns [w*DW, (w+1)*DW) --------------
  float acc[MT][NTO][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int jn = 0; jn < NTO; ++jn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][jn][e] = 0.f;
  // keys in steps of 16, then one step of 8 when KP is not a multiple of 16
  for (int kk = 0; kk < KP / 16; ++kk) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int row = mt * 16 + (lane & 15);
      const int col = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(sP + (row * LDP + col) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
    }
    const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
    if (NTO >= 2) {
#pragma unroll
      for (int jp = 0; jp < NTO / 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int col = warp * DW + jp * 16 + (lane >> 4) * 8;
        ldsm_x4_t(sw128_addr(sV, KP, key, col), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_16816(acc[mt][2 * jp], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
          mma_16816(acc[mt][2 * jp + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
        }
      }
    } else {
      uint32_t b0, b1;
      ldsm_x2_t(sw128_addr(sV, KP, key, warp * DW), b0, b1);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        mma_16816(acc[mt][0], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
    }
  }
  if (KP % 16 == 8) {
    const int k0 = KP - 8;
    uint32_t a[MT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
      ldsm_x2(sP + ((mt * 16 + (lane & 15)) * LDP + k0) * 2, a[mt][0], a[mt][1]);
#pragma unroll
    for (int jn = 0; jn < NTO; ++jn) {
      uint32_t b0;
      ldsm_x1_t(sw128_addr(sV, KP, k0 + (lane & 7), warp * DW + jn * 8), b0);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) mma_1688(acc[mt][jn], a[mt][0], a[mt][1], b0);
    }
  }

  // ---- O / l -> bf16 into a swizzled staging tile (K/V's buffer, free once
  // every warp is past PV), then one TMA box store per 64 columns ----------
  __syncthreads();
  const uint32_t sO = sK;  // NCH blocks of [32 rows][128 bytes]
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      if (trow[mt][hf] >= 0) {
        const float inv_l = 1.f / row_l[row];
#pragma unroll
        for (int jn = 0; jn < NTO; ++jn) {
          const int col = warp * DW + jn * 8;
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sw128_addr(sO, 32, row, col) +
                                                        4 * (lane & 3)),
                       "r"(pack_bf16x2(acc[mt][jn][2 * hf] * inv_l,
                                       acc[mt][jn][2 * hf + 1] * inv_l))
                       : "memory");
        }
      }
    }
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) tma_store_4d(&tm_o, sO + ch * 32 * 128, ch * 64, g * G, 0, b);
    tma_store_commit();
    tma_store_wait_read<0>();  // the staging tile is read before the CTA leaves
  }
}

// Copy accepted new tokens into their ring slots: block = (sequence, token).
__global__ void __launch_bounds__(128)
    kv_commit_kernel(__nv_bfloat16* k_ring, __nv_bfloat16* v_ring,
                     const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                     const int32_t* pos, const int32_t* n_accept, int n_q, int Hkv, int D,
                     int W) {
  const int b = blockIdx.x / n_q;
  const int u = blockIdx.x - b * n_q;
  int na = __ldg(n_accept + b);
  const int P = __ldg(pos + b);
  if (na < 0 || na > n_q || P < 0) {
    if (u == 0 && threadIdx.x == 0) flag_error(2u);
    if (P < 0) return;
    na = min(max(na, 0), n_q);
  }
  if (u >= na) return;
  const int64_t slot = (static_cast<int64_t>(P) + u) % W;
  const int n16 = Hkv * D / 8;  // 16-byte chunks per token (all kv heads)
  const uint4* ks = reinterpret_cast<const uint4*>(k_new + (static_cast<size_t>(b) * n_q + u) * Hkv * D);
  const uint4* vs = reinterpret_cast<const uint4*>(v_new + (static_cast<size_t>(b) * n_q + u) * Hkv * D);
  uint4* kd = reinterpret_cast<uint4*>(k_ring + (static_cast<size_t>(b) * W + slot) * Hkv * D);
  uint4* vd = reinterpret_cast<uint4*>(v_ring + (static_cast<size_t>(b) * W + slot) * Hkv * D);
  for (int idx = threadIdx.x; idx < n16; idx += blockDim.x) {
    kd[idx] = ks[idx];
    vd[idx] = vs[idx];
  }
}

}  // namespace swa
