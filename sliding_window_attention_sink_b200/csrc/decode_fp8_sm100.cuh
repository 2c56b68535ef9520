// decode_fp8_sm100.cuh -- decode / draft verification over a W-slot ring of
// FP8 (E4M3) codes, and the commit of accepted tokens into such a ring.
//
// Operation: exactly the decode of decode_sm100.cuh over the ring values
// code value x scale, with one fp32 scale per kv head for K and one for V.
// The KV cache of these models is sized as an FP8 cache (MiMo-V3 / HySparse2
// news page, cost comparison at one million tokens), and inference runs in
// FP8 with the E4M3 format (MiMo-V2 blog review, sections 4.3 and 6). The
// ring's bytes halve; Q, the new tokens and O stay bf16.
//
// Design (sm_100a), one CTA per (sequence, kv head) as for the bf16 ring:
// * Every load is issued at the start by one thread as TMA boxes: Q and the
//   new K and V rows (bf16, 128-byte swizzle) and the K and V codes, one box
//   of W rows x D bytes each, swizzled (128 bytes for D = 128, 64 for D = 64)
//   so that the fragment loads below meet distinct banks. The codes are read
//   straight from these staging tiles: no bf16 copy of the ring is made, so
//   four CTAs share an SM with ~44 KB each in flight.
// * The contractions run on mma.sync m16n8k16 with f16 operands and f32
//   accumulation: one cvt turns two E4M3 codes into an f16 pair, exactly
//   (every E4M3 value is an f16 normal number). The codes are used by only
//   the 32 query rows of the CTA, so a conversion of several instructions
//   per pair (to bf16) would dominate the kernel. Q is converted to f16 once,
//   in place in shared memory: exact for |q| in [2^-14, 65504]; smaller
//   magnitudes round to the f16 subnormal grid (absolute error <= 2^-25),
//   larger ones saturate to 65504. P is rounded to f16 (finer than bf16 on
//   [0, 1]); the new tokens' bf16 K and V rows are converted to f16 as their
//   fragments are loaded.
// * S = Q K^T: the order of the 16 head-dim columns of each k-step is
//   permuted alike in Q and K (logical 2c, 2c+1, 2c+8, 2c+9 <-> stored
//   4c .. 4c+3). An ldmatrix over the code tile hands each thread 4
//   consecutive codes of one key row per 8x8 (16-bit) matrix, i.e. both of
//   its K fragment registers; one ldmatrix.x4 covers four k-steps. Q is
//   stored reordered (in its f16 conversion) so that plain ldmatrix A
//   fragments come out in the same order.
// * O = P V: an ldmatrix over the V code tile gives a thread 4 codes of one
//   key row (stored head-dim columns 4c .. 4c+3 of a 16-column group); they
//   become two f16 pairs, and movmatrix transposes each 8x8 tile into the B
//   fragment. The two tiles of a group hold the stored columns {4c, 4c+1}
//   and {4c+2, 4c+3}, which the epilogue writes back in place.
// * K's scale multiplies the logits of the ring columns. V's scale is applied
//   in fp32: the new tokens (a 16-key block of their own: the ring's columns
//   are padded to a multiple of 16) are accumulated first, the accumulator
//   is divided by the scale, the ring's blocks follow, and O is multiplied by
//   the scale at the end.
// * The V rows of never-written slots (pos < W) and of the padding are set
//   to zero codes in shared memory, so NaN bytes there cannot reach O.
#pragma once
#include "decode_sm100.cuh"

namespace swa {

struct DecodeFp8Params : DecodeParams {
  const float* kv_scale;  // [2 * Hkv]: K scales, then V scales
};

__host__ __device__ inline size_t round1024(size_t x) { return (x + 1023) / 1024 * 1024; }

// Shared memory (from a 1024-byte aligned base): Q [D/64][32 rows][128 B]
// (later P [32][KP+8] bf16, then the O staging tile); the K and V code tiles
// [W8 rows][D bytes] (swizzled); the new K and V rows [D/64][16 rows][128 B];
// per-warp row maxima and row sums [NWP][32] and row l [32] (fp32).
__host__ __device__ inline size_t decode_fp8_smem_bytes(int D, int KP, int W8, int nwp) {
  return 1024 + round1024(decode_qp_bytes(D, KP)) + 2 * round1024(static_cast<size_t>(W8) * D) +
         2 * static_cast<size_t>(D / 64) * 2048 +
         (static_cast<size_t>(nwp) * 32 * 2 + 32) * sizeof(float);
}

// Byte address of (row, byte) in a code tile of D-byte rows written by TMA
// with the 128-byte (D = 128) or 64-byte (D = 64) swizzle: 16-byte unit bits
// 4.. of the offset XOR its bits 7.. (3 bits for 128, 2 for 64).
template <int D>
__device__ __forceinline__ uint32_t code_addr(uint32_t base, int row, int byte) {
  const uint32_t off = static_cast<uint32_t>(row * D + byte);
  constexpr uint32_t kMask = D == 128 ? 7u : 3u;
  return base + (off ^ (((off >> 7) & kMask) << 4));
}

// Four E4M3 codes (bytes 0..3 of w) -> f16 pairs {0, 1} and {2, 3}, exactly.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 c01, c23;\n\t"
      "mov.b32 {c01, c23}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, c01;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}
// bf16 pair -> f16 pair (round to nearest; beyond 65504 saturated).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;"
      : "=r"(r)
      : "f"(bf16hi_to_f32(x)), "f"(bf16lo_to_f32(x)));
  return r;
}
// bf16 pair x s -> f16 pair (round to nearest; beyond 65504 saturated).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t x, float s) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;"
      : "=r"(r)
      : "f"(bf16hi_to_f32(x) * s), "f"(bf16lo_to_f32(x) * s));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// A shared-memory read as a plain load (not asm), so that the compiler may
// schedule it ahead of the conversions and MMAs of earlier tiles; the
// barrier waits (asm with a memory clobber) keep it after the data lands.
// (smem: the dynamic shared array; addr: a shared-window address in it)
__device__ __forceinline__ void lds64(const uint8_t* smem, uint32_t addr, uint32_t& lo,
                                      uint32_t& hi) {
  const uint2 v = *reinterpret_cast<const uint2*>(smem + (addr - smem_u32(smem)));
  lo = v.x;
  hi = v.y;
}
// mma.sync m16n8k16 f16 -> f32 as a pure register operation (no volatile)
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}
// Byte address of bf16 column `col` (a multiple of 4) of `row` in a
// 128-byte-swizzled tile of `rows` rows per 64-column block.
__device__ __forceinline__ uint32_t bf16_addr(uint32_t base, int rows, int row, int col) {
  return sw128_addr(base, rows, row, col & ~7) + (col & 7) * 2;
}

template <int D, int MT, int NWP>
__global__ void __launch_bounds__(NWP * 32, NWP == kDecodeSmallWarps ? 4 : 2)
    decode_fp8_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k8,
                            const __grid_constant__ CUtensorMap tm_kn,
                            const __grid_constant__ CUtensorMap tm_v8,
                            const __grid_constant__ CUtensorMap tm_vn,
                            const __grid_constant__ CUtensorMap tm_o,
                            const DecodeFp8Params p) {
  constexpr int NT_ = NWP * 32;
  constexpr int NCH = D / 64;      // 64-column blocks of the head dim
  constexpr int RP = MT * 16;      // padded query rows
  constexpr int NTW = 5;           // max n8 key tiles per warp (KP <= 40 * NWP)
  constexpr int DW = D / NWP;      // PV: head-dim columns per warp (8, 16 or 32)
  constexpr int NTO = DW / 8;      // n8 tiles per warp in PV
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_qk, bar_v;
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;
  const int KP = p.KP, W = p.W, W8 = p.W8, n_q = p.n_q, G = p.G;
  const uint32_t sQ = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint8_t* sm = smem_raw;
  const uint32_t sK8 = sQ + static_cast<uint32_t>(round1024(decode_qp_bytes(D, KP)));
  const uint32_t ring_bytes = static_cast<uint32_t>(round1024(static_cast<size_t>(W8) * D));
  const uint32_t sV8 = sK8 + ring_bytes;
  const uint32_t sKn = sV8 + ring_bytes;  // [NCH][16 rows][128 B]
  const uint32_t sVn = sKn + NCH * 2048;
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(smem_raw + (sQ - smem_u32(smem_raw)));
  const int LDP = KP + 8;
  float* red_max = reinterpret_cast<float*>(smem_raw + (sVn + NCH * 2048 - smem_u32(smem_raw)));
  float* red_lx = red_max + NWP * 32;  // [NWP][32]
  float* row_l = red_lx + NWP * 32;    // [32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, c4 = lane & 3;  // fragment row / column pair
  const int b = blockIdx.x / p.Hkv;
  const int g = blockIdx.x - b * p.Hkv;

  // ---- every load, issued at once by one thread ------------------------------
  if (tid == 0) {
    mbar_init(smem_u32(&bar_qk), 1);
    mbar_init(smem_u32(&bar_v), 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k8);
    tma_prefetch_desc(&tm_kn);
    tma_prefetch_desc(&tm_v8);
    tma_prefetch_desc(&tm_vn);
    const uint32_t side = W * D + NCH * n_q * 128;  // codes + new rows
    mbar_arrive_expect_tx(smem_u32(&bar_qk), NCH * p.R * 128 + side);
    tma_load_4d(sK8, &tm_k8, smem_u32(&bar_qk), 0, g, 0, b);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      tma_load_4d(sQ + ch * 32 * 128, &tm_q, smem_u32(&bar_qk), ch * 64, g * G, 0, b);
      tma_load_4d(sKn + ch * 2048, &tm_kn, smem_u32(&bar_qk), ch * 64, g, 0, b);
    }
    mbar_arrive_expect_tx(smem_u32(&bar_v), side);
    tma_load_4d(sV8, &tm_v8, smem_u32(&bar_v), 0, g, 0, b);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
      tma_load_4d(sVn + ch * 2048, &tm_vn, smem_u32(&bar_v), ch * 64, g, 0, b);
  }

  // V's padding rows W .. W8-1 (no box writes them) hold zero codes: P is 0
  // there, and 0 * V must stay 0
  for (int idx = tid; idx < (W8 - W) * (D / 16); idx += NT_)
    *reinterpret_cast<uint4*>(smem_raw + (sV8 + W * D + idx * 16 - smem_u32(smem_raw))) =
        make_uint4(0u, 0u, 0u, 0u);

  // ---- this thread's rows, sinks and scales (while the loads fly) ------------
  int P = __ldg(p.pos + b);
  if (P < 0) {
    if (tid == 0) flag_error(2u);
    P = 0;
  }
  // Key ranks as for the bf16 ring: slot s has rank (s - P) mod W, new token
  // u rank W + u; query t sees the ranks [max(t + 1, W - P), W + t].
  const int Pmod = P % W;
  int trow[MT][2], rlo[MT][2];
  unsigned rspan[MT][2];
  float srow[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + gq + hf * 8;
      const int t = row < p.R ? row / G : -1;  // -1: padding row, sees nothing
      trow[mt][hf] = t;
      rlo[mt][hf] = t >= 0 ? max(t + 1, W - P) : 0x7fffffff;
      rspan[mt][hf] = t >= 0 ? static_cast<unsigned>(W + t - rlo[mt][hf]) : 0u;
      srow[mt][hf] = (t >= 0 && p.sink != nullptr)
                         ? __ldg(p.sink + g * G + (row - t * G)) * kLog2e
                         : -INFINITY;
    }
  float sk_tid = -INFINITY;
  if (tid < p.R && p.sink != nullptr) {
    const int t = tid / G;
    sk_tid = __ldg(p.sink + g * G + (tid - t * G)) * kLog2e;
  }
  const float k_sc = __ldg(p.kv_scale + g), v_sc = __ldg(p.kv_scale + p.Hkv + g);
  if (tid == 0 && !(k_sc > 0.f && v_sc > 0.f && k_sc < INFINITY && v_sc < INFINITY))
    flag_error(2u);
  const float sc_ring = p.scale_log2 * k_sc;

  if (!__syncthreads_and(mbar_wait(smem_u32(&bar_qk), 0, abort))) return;
  // Q (bf16) -> f16 in place, each 16-column group reordered so that the
  // standard ldmatrix A fragments come out in the permuted column order:
  // stored pairs 0..3 <- columns {4c, 4c+1}, pairs 4..7 <- {4c+2, 4c+3}.
  for (int gi = tid; gi < NCH * 32 * 4; gi += NT_) {
    const int row = (gi >> 2) & 31, ch = gi >> 7, grp = gi & 3;
    const uint32_t blk = sQ + ch * 32 * 128 + row * 128;
    uint8_t* u0 = smem_raw + (blk + (((2 * grp) ^ (row & 7)) << 4) - smem_u32(smem_raw));
    uint8_t* u1 = smem_raw + (blk + (((2 * grp + 1) ^ (row & 7)) << 4) - smem_u32(smem_raw));
    const uint4 x = *reinterpret_cast<const uint4*>(u0), y = *reinterpret_cast<const uint4*>(u1);
    *reinterpret_cast<uint4*>(u0) = make_uint4(bf16x2_to_f16x2(x.x), bf16x2_to_f16x2(x.z),
                                               bf16x2_to_f16x2(y.x), bf16x2_to_f16x2(y.z));
    *reinterpret_cast<uint4*>(u1) = make_uint4(bf16x2_to_f16x2(x.y), bf16x2_to_f16x2(x.w),
                                               bf16x2_to_f16x2(y.y), bf16x2_to_f16x2(y.w));
  }
  __syncthreads();

  // ---- S = Q K^T: warp w takes key tiles w, w + NWP, ... ----------------------
  // Tiles at or past NTS hold padding only: no S, and P = 0 there. The new
  // keys are divided by K's scale as they are converted, so that every
  // column's logit is S x sc_ring.
  const int NT = KP / 8, NTS = (W8 + n_q + 7) / 8;
  const float k_inv = 1.f / k_sc;
  float s[MT][NTW][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[mt][j][e] = 0.f;
  // four k-steps at a time: Q's A fragments of the four (ldmatrix), then per
  // key tile the codes of the four (one ldmatrix.x4: matrix i = rows of the
  // tile x the 16 codes of k-step i, 4 codes per thread) or the new rows
#pragma unroll
  for (int kq = 0; kq < D / 64; ++kq) {
    uint32_t a[4][MT][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int row = mt * 16 + (lane & 15);
        const int col = (kq * 4 + i) * 16 + (lane >> 4) * 8;
        ldsm_x4(sw128_addr(sQ, 32, row, col), a[i][mt][0], a[i][mt][1], a[i][mt][2],
                a[i][mt][3]);
      }
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      const int nt = warp + NWP * j;
      if (nt < NTS) {
        uint32_t b[4][2];
        if (nt * 8 < W8) {  // ring keys: codes
          uint32_t w[4];
          ldsm_x4(code_addr<D>(sK8, nt * 8 + (lane & 7), (kq * 4 + (lane >> 3)) * 16), w[0], w[1],
                  w[2], w[3]);
#pragma unroll
          for (int i = 0; i < 4; ++i) e4m3x4_to_f16x2(w[i], b[i][0], b[i][1]);
        } else {  // new keys: bf16 rows
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            lds64(sm, bf16_addr(sKn, 16, nt * 8 - W8 + gq, (kq * 4 + i) * 16 + 4 * c4), b[i][0],
                  b[i][1]);
            b[i][0] = bf16x2_to_f16x2_scaled(b[i][0], k_inv);
            b[i][1] = bf16x2_to_f16x2_scaled(b[i][1], k_inv);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            mma_f16_16816(s[mt][j], a[i][mt][0], a[i][mt][1], a[i][mt][2], a[i][mt][3], b[i][0],
                          b[i][1]);
      }
    }
  }

  // ---- mask (raw logits) and per-warp row max -------------------------------
  // The scale sc_ring > 0 goes into the exponent below. A ring tile whose
  // slots all have rank >= thr = max(n_q, W - P) is seen whole by every query
  // row (query t hides ranks < max(t + 1, W - P)): a warp vote skips its mask.
  const int thr = max(n_q, W - P);
  float mloc[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) mloc[mt][0] = mloc[mt][1] = -INFINITY;
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    const int nt = warp + NWP * j;
    if (nt >= NTS) continue;  // warp-uniform
    int rank[2];
    bool hidden = false;
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int col = nt * 8 + 2 * c4 + e2;
      rank[e2] = 0x3fffffff;  // padding: seen by no query
      if (col < W) {
        rank[e2] = col - Pmod;
        if (rank[e2] < 0) rank[e2] += W;
      } else if (col >= W8 && col < W8 + n_q) {
        rank[e2] = W + (col - W8);
      }
      hidden |= rank[e2] < thr || rank[e2] >= W;
    }
    if (!__any_sync(0xffffffffu, hidden)) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          mloc[mt][hf] = max3(mloc[mt][hf], s[mt][j][hf * 2], s[mt][j][hf * 2 + 1]);
      continue;
    }
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2)
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const bool vis = static_cast<unsigned>(rank[e2] - rlo[mt][hf]) <= rspan[mt][hf];
          float& x = s[mt][j][hf * 2 + e2];
          x = vis ? x : -INFINITY;
          mloc[mt][hf] = fmaxf(mloc[mt][hf], x);
        }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v = mloc[mt][hf];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
      if (c4 == 0) red_max[warp * 32 + mt * 16 + gq + hf * 8] = v;
    }
  __syncthreads();

  // ---- row max over warps and the sink (log2 units); P = exp2(x sc - m) ->
  // smem (f16); row sums of the unrounded P (f16 P is close enough that O
  // needs no sum of the rounded weights) ------------------------------------
  float mrow[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + gq + hf * 8;
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < NWP; ++w) m = fmaxf(m, red_max[w * 32 + row]);
      m = fmaxf(srow[mt][hf], m * sc_ring);
      mrow[mt][hf] = (m == -INFINITY) ? 0.f : m;
    }
  float lx[MT][2];
  const uint32_t sP = smem_u32(Ps);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    lx[mt][0] = lx[mt][1] = 0.f;
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      const int nt = warp + NWP * j;
      if (nt < NT) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int row = mt * 16 + gq + hf * 8;
          const int col = nt * 8 + 2 * c4;
          uint32_t pk = 0u;
          if (nt < NTS) {
            const float p0 = ex2(fmaf(s[mt][j][2 * hf], sc_ring, -mrow[mt][hf]));
            const float p1 = ex2(fmaf(s[mt][j][2 * hf + 1], sc_ring, -mrow[mt][hf]));
            pk = pack_f16x2(p0, p1);
            lx[mt][hf] += p0 + p1;
          }
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
      float x = lx[mt][hf];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (c4 == 0) red_lx[warp * 32 + mt * 16 + gq + hf * 8] = x;
    }
  // V's codes and new rows in shared memory; a wait that gave up ends every
  // thread here (the barrier also publishes P and the row sums)
  if (!__syncthreads_and(mbar_wait(smem_u32(&bar_v), 0, abort))) return;
  // with fewer than W committed tokens the slots P .. W-1 were never written
  // and may hold anything (NaN codes too): zero codes there
  if (P < W) {
    for (int idx = tid; idx < (W - P) * (D / 16); idx += NT_)
      *reinterpret_cast<uint4*>(smem_raw + (sV8 + P * D + idx * 16 - smem_u32(smem_raw))) =
          make_uint4(0u, 0u, 0u, 0u);
  }
  if (tid < RP) {
    const int row = tid;
    const int t = row < p.R ? row / G : -1;
    const float sk = sk_tid;
    float m = -INFINITY;
    for (int w = 0; w < NWP; ++w) m = fmaxf(m, red_max[w * 32 + row]);
    m = fmaxf(sk, m * sc_ring);
    const float mb = (m == -INFINITY) ? 0.f : m;
    float lxs = 0.f;
    for (int w = 0; w < NWP; ++w) lxs += red_lx[w * 32 + row];
    if (sk != -INFINITY) lxs += ex2(sk - mb);
    row_l[row] = lxs;
    if (t >= 0 && p.lse != nullptr)
      p.lse[(static_cast<size_t>(b) * n_q + t) * p.Hq + g * G + (row - t * G)] =
          (mb + lg2(lxs)) * kLn2;
  }

  // ---- O = P V: warp w takes stored head-dim columns [w*DW, (w+1)*DW) --------
  // Ring rows at or past min(P, W) (never written, or padding) hold zero
  // codes (see above) and new rows past n_q read as zero. W8 (the first
  // new-token column) is a multiple of 16 here, and the new tokens fill the
  // one block after it.
  float acc[MT][NTO][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int jn = 0; jn < NTO; ++jn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][jn][e] = 0.f;
  // stored columns of this thread's fragment row in each 16-column group
  constexpr int NGRP = DW >= 16 ? DW / 16 : 1;
  const int gbase = DW >= 16 ? warp * DW : (warp >> 1) * 16;
  // one 16-key block: P's A fragments, the B fragments of the warp's
  // columns (codes of ring keys, or the new tokens' bf16 rows), the MMAs
  auto pv_block = [&](int kb, bool ring) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int row = mt * 16 + (lane & 15);
      const int col = kb * 16 + (lane >> 4) * 8;
      ldsm_x4(sP + (row * LDP + col) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
    }
    // ring codes: one ldmatrix for the warp's columns (matrix i: key half
    // i & 1 of the block x the 16 codes of group i >> 1)
    uint32_t vw[NGRP][2];
    if (ring) {
      const uint32_t va = code_addr<D>(sV8, kb * 16 + 8 * ((lane >> 3) & 1) + (lane & 7),
                                       gbase + (NGRP == 2 ? (lane >> 4) : 0) * 16);
      if constexpr (NGRP == 2)
        ldsm_x4(va, vw[0][0], vw[0][1], vw[NGRP - 1][0], vw[NGRP - 1][1]);
      else
        ldsm_x2(va, vw[0][0], vw[0][1]);
    }
#pragma unroll
    for (int q = 0; q < NGRP; ++q) {
      const int col = gbase + q * 16 + 4 * c4;
      uint32_t fa[2], fb[2];  // row fragments of the two 8x8 tiles, key halves 0 / 1
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int key = kb * 16 + 8 * h + gq;
        if (ring) {
          e4m3x4_to_f16x2(vw[q][h], fa[h], fb[h]);
        } else if (key - W8 < n_q) {
          lds64(sm, bf16_addr(sVn, 16, key - W8, col), fa[h], fb[h]);
          fa[h] = bf16x2_to_f16x2(fa[h]);
          fb[h] = bf16x2_to_f16x2(fb[h]);
        } else {
          fa[h] = fb[h] = 0u;
        }
      }
      if constexpr (DW >= 16) {
        const uint32_t a0 = movmatrix_t(fa[0]), a1 = movmatrix_t(fa[1]);
        const uint32_t b0 = movmatrix_t(fb[0]), b1 = movmatrix_t(fb[1]);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_f16_16816(acc[mt][2 * q], a[mt][0], a[mt][1], a[mt][2], a[mt][3], a0, a1);
          mma_f16_16816(acc[mt][2 * q + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
        }
      } else {  // one tile per warp: the even warp of a pair takes {4c, 4c+1}
        const bool second = warp & 1;
        const uint32_t t0 = movmatrix_t(second ? fb[0] : fa[0]);
        const uint32_t t1 = movmatrix_t(second ? fb[1] : fa[1]);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          mma_f16_16816(acc[mt][0], a[mt][0], a[mt][1], a[mt][2], a[mt][3], t0, t1);
      }
    }
  };
  if (P < W) __syncthreads();  // the zeroed rows (a CTA-uniform condition)
  // the new tokens first (unscaled V), then acc / v_sc, then the ring's codes
  pv_block(W8 / 16, false);
  {
    const float v_inv = 1.f / v_sc;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int jn = 0; jn < NTO; ++jn)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][jn][e] *= v_inv;
  }
#pragma unroll 1
  for (int kb = 0; kb < W8 / 16; ++kb) pv_block(kb, true);

  // ---- O * v_sc / l -> bf16 into the staging tile over Q / P, then one TMA box
  // store per 64 columns --------------------------------------------------------
  __syncthreads();
  const uint32_t sO = sQ;  // NCH blocks of [32 rows][128 bytes]
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + gq + hf * 8;
      if (trow[mt][hf] >= 0) {
        const float f = v_sc / row_l[row];
        if constexpr (DW >= 16) {
#pragma unroll
          for (int q = 0; q < NGRP; ++q) {
            const uint32_t lo = pack_bf16x2(acc[mt][2 * q][2 * hf] * f, acc[mt][2 * q][2 * hf + 1] * f);
            const uint32_t hi =
                pack_bf16x2(acc[mt][2 * q + 1][2 * hf] * f, acc[mt][2 * q + 1][2 * hf + 1] * f);
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(
                             bf16_addr(sO, 32, row, gbase + q * 16 + 4 * c4)),
                         "r"(lo), "r"(hi)
                         : "memory");
          }
        } else {
          const int col = gbase + 4 * c4 + ((warp & 1) ? 2 : 0);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(bf16_addr(sO, 32, row, col)),
                       "r"(pack_bf16x2(acc[mt][0][2 * hf] * f, acc[mt][0][2 * hf + 1] * f))
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

// Two floats -> two E4M3 codes (lo in the low byte): round to nearest even,
// magnitudes beyond 448 saturated.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// FP8 ring commit: accepted token u of sequence b goes to slot (pos + u) mod
// W as the E4M3 codes of x / scale (the quotient rounded to fp32 by IEEE
// division). Block = (sequence, token); thread = 8 values of K and of V.
__global__ void __launch_bounds__(128)
    kv_commit_fp8_kernel(uint8_t* k_ring, uint8_t* v_ring, const __nv_bfloat16* k_new,
                         const __nv_bfloat16* v_new, const float* kv_scale,
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
  const int n8 = Hkv * D / 8;  // 8-value chunks per token (all kv heads)
  const size_t src = (static_cast<size_t>(b) * n_q + u) * Hkv * D;
  const size_t dst = (static_cast<size_t>(b) * W + slot) * Hkv * D;
  const uint4* ks = reinterpret_cast<const uint4*>(k_new + src);
  const uint4* vs = reinterpret_cast<const uint4*>(v_new + src);
  uint2* kd = reinterpret_cast<uint2*>(k_ring + dst);
  uint2* vd = reinterpret_cast<uint2*>(v_ring + dst);
  for (int idx = threadIdx.x; idx < n8; idx += blockDim.x) {
    const int gh = idx * 8 / D;
    const float sk = __ldg(kv_scale + gh), sv = __ldg(kv_scale + Hkv + gh);
    if (!(sk > 0.f && sv > 0.f && sk < INFINITY && sv < INFINITY)) flag_error(2u);
    const uint4 kx = ks[idx], vx = vs[idx];
    const uint32_t kw[4] = {kx.x, kx.y, kx.z, kx.w}, vw[4] = {vx.x, vx.y, vx.z, vx.w};
    uint32_t ko[2], vo[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ko[h] = f32x2_to_e4m3x2(__fdiv_rn(bf16lo_to_f32(kw[2 * h]), sk),
                              __fdiv_rn(bf16hi_to_f32(kw[2 * h]), sk)) |
              (f32x2_to_e4m3x2(__fdiv_rn(bf16lo_to_f32(kw[2 * h + 1]), sk),
                               __fdiv_rn(bf16hi_to_f32(kw[2 * h + 1]), sk))
               << 16);
      vo[h] = f32x2_to_e4m3x2(__fdiv_rn(bf16lo_to_f32(vw[2 * h]), sv),
                              __fdiv_rn(bf16hi_to_f32(vw[2 * h]), sv)) |
              (f32x2_to_e4m3x2(__fdiv_rn(bf16lo_to_f32(vw[2 * h + 1]), sv),
                               __fdiv_rn(bf16hi_to_f32(vw[2 * h + 1]), sv))
               << 16);
    }
    kd[idx] = make_uint2(ko[0], ko[1]);
    vd[idx] = make_uint2(vo[0], vo[1]);
  }
}

}  // namespace swa
