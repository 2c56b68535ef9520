// decode_splitkv_sm100.cuh -- decode / draft verification over a long KV
// cache (the global-attention layers), split over the cached positions.
//
// Operation: the sink attention of "MiMo-V2-Flash Technical Report" summary
// (mlpod.com), section 2.2.2, for the decode step of the global-attention
// layers of section 2.2 (every earlier token visible), with the verification
// of MTP drafts of section 2.3 (n_q new tokens, causal among themselves). The
// cache follows the same convention as the W-slot ring of the sliding-window
// decode: the token at position p sits in slot p mod W, and query t (absolute
// position P + t) sees the cached positions max(0, P + t - W + 1) .. P - 1
// and the new tokens 0 .. t. With W at least the context length the cache is
// a plain array indexed by position and every earlier token is visible.
//
// Split-KV ("flash decoding"): the cached positions of a (sequence, kv head)
// are cut into S ranges of `chunk` positions; one CTA per range streams its
// K/V in 64-key tiles through a 3-stage TMA pipeline, keeps an online softmax
// over them (max in log2 units, unnormalised O, two row sums) and writes that
// partial state. The last range also takes the n_q new tokens, as one more
// tile through the same pipeline. A second
// kernel merges the S partial states of each row and adds the sink term once:
//   M = max(s, max_r m_r),  O = sum_r 2^(m_r - M) O_r / L,
//   L = sum_r 2^(m_r - M) l_r + 2^(s - M),  LSE = (M + log2(same with l_x)) ln 2.
//
// Per CTA: 4 warps; R = n_q * G query rows (<= 32) as the M dimension of
// mma.sync m16n8k16 (the tiles are too small for tcgen05); warp w takes keys
// [16 w, 16 w + 16) of a tile for S and head-dim columns [w D/4, (w+1) D/4)
// for O = P V. Row maxima cross the warps through shared memory.
//
// Every wait is bounded (see mbar_wait); nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kSplitWarps = 4;
constexpr int kSplitTile = 64;    // keys per tile
constexpr int kSplitStages = 3;   // K/V tiles in flight (two CTAs per SM at D = 128)

struct SplitParams {
  const int32_t* pos;
  int B, n_q, Hq, Hkv, G, W, R;
  int S;          // ranges per (sequence, kv head)
  int chunk;      // cached positions per range (a multiple of kSplitTile)
  const float* sink;
  float scale_log2;
  float* part;    // [B * Hkv * S][32 rows][D + 4]: O (unnormalised), m, l_r, l_x
  __nv_bfloat16* o;
  float* lse;
};

// Shared memory (1024-byte aligned base): kSplitStages stages of K and V tiles
// (D/64 blocks of [64 rows][128 bytes] each, 128-byte swizzle), Q (D/64 blocks
// of [32 rows][128 bytes]), P [32][kSplitTile + 8] bf16, the row exchange
// [4][32] fp32.
__host__ __device__ inline size_t split_smem_bytes(int D) {
  const size_t nch = D / 64;
  const size_t tile = nch * kSplitTile * 128;
  return 1024 + 2 * kSplitStages * tile + nch * 32 * 128 +
         static_cast<size_t>(32) * (kSplitTile + 8) * 2 + 4 * 32 * sizeof(float);
}

template <int D, int MT>
__global__ void __launch_bounds__(kSplitWarps * 32, 2)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_kc,
                        const __grid_constant__ CUtensorMap tm_vc,
                        const __grid_constant__ CUtensorMap tm_kn,
                        const __grid_constant__ CUtensorMap tm_vn, const SplitParams p) {
  constexpr int NCH = D / 64;
  constexpr int RP = MT * 16;                   // padded query rows
  constexpr int T = kSplitTile;
  constexpr uint32_t TILE = NCH * T * 128;      // bytes of one K or V tile
  constexpr int DW = D / kSplitWarps;           // PV head-dim columns per warp
  constexpr int NTO = DW / 8;                   // n8 tiles per warp in PV (2 or 4)
  constexpr int LDP = T + 8;                    // P row stride (bf16 elements)
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, full[kSplitStages];
  __shared__ int abort_sh;
  volatile int* abort = &abort_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTAs that run together take the same positions of all kv heads of a
  // sequence (blockIdx = (b * S + s) * Hkv + g): a cached token's rows of the
  // Hkv heads are adjacent in HBM and are then fetched at about the same time
  const int bs = blockIdx.x / p.Hkv, g = blockIdx.x - bs * p.Hkv;
  const int b = bs / p.S, s = bs - b * p.S;
  const int unit = (b * p.Hkv + g) * p.S + s;  // partial-state slot
  const int W = p.W, n_q = p.n_q, G = p.G;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sKs = base;  // stage st: K at sKs + st * 2 * TILE, V TILE further
  const uint32_t sQ = base + 2 * kSplitStages * TILE;
  uint8_t* gen = smem_raw + (sQ + NCH * 32 * 128 - smem_u32(smem_raw));
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(gen);
  float* red = reinterpret_cast<float*>(gen + 32 * LDP * 2);  // [4][32]

  if (tid == 0) {
    mbar_init(smem_u32(&bar_q), 1);
    for (int i = 0; i < kSplitStages; ++i) mbar_init(smem_u32(&full[i]), 1);
    abort_sh = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // this range of cached positions: [r0, r1), tiles aligned to T positions
  int P = __ldg(p.pos + b);
  if (P < 0) {
    if (tid == 0 && s == 0) flag_error(2u);
    P = 0;
  }
  const int lo0 = max(0, P - W + 1);  // oldest position any query of b sees
  const int r0 = lo0 + s * p.chunk;
  const int r1 = min(r0 + p.chunk, P);
  if (s == p.S - 1 && r1 < P && tid == 0) flag_error(2u);  // pos beyond the split cover
  const int t0 = (r0 / T) * T;                      // first tile start
  const int ntile = r1 > r0 ? (r1 - t0 + T - 1) / T : 0;
  const bool last = s == p.S - 1;                   // also takes the new tokens
  const int nall = ntile + (last ? 1 : 0);          // tiles through the pipeline

  // loads: Q (and the new tokens) once; K/V tiles through the stages
  // tile i -> stage i % kSplitStages: cached positions, or for i == ntile the
  // n_q new tokens in rows 0 .. n_q-1
  auto issue_tile = [&](int i) {
    const int st = i % kSplitStages;
    const uint32_t bar = smem_u32(&full[st]);
    const uint32_t dk = sKs + st * 2 * TILE, dv = dk + TILE;
    if (i < ntile) {
      const int slot = (t0 + i * T) % W;  // W % T == 0: a tile never wraps
      mbar_arrive_expect_tx(bar, 2 * TILE);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        tma_load_4d(dk + ch * T * 128, &tm_kc, bar, ch * 64, g, slot, b);
        tma_load_4d(dv + ch * T * 128, &tm_vc, bar, ch * 64, g, slot, b);
      }
    } else {
      mbar_arrive_expect_tx(bar, 2 * NCH * n_q * 128);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        tma_load_4d(dk + ch * T * 128, &tm_kn, bar, ch * 64, g, 0, b);
        tma_load_4d(dv + ch * T * 128, &tm_vn, bar, ch * 64, g, 0, b);
      }
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_kc);
    tma_prefetch_desc(&tm_vc);
    mbar_arrive_expect_tx(smem_u32(&bar_q), NCH * p.R * 128);
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
      tma_load_4d(sQ + ch * 32 * 128, &tm_q, smem_u32(&bar_q), ch * 64, g * G, 0, b);
    for (int i = 0; i < min(nall, kSplitStages); ++i) issue_tile(i);
  }

  // this thread's rows: fragment rows lane/4 and lane/4 + 8 of each m-tile
  int trow[MT][2], vlo[MT][2];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      const int t = row < p.R ? row / G : -1;
      trow[mt][hf] = t;
      // first cached position the row sees within this range
      vlo[mt][hf] = t >= 0 ? max(r0, max(0, P + t - W + 1)) : 0x7fffffff;
    }

  float m_run[MT][2], lr[MT][2], lx[MT][2];
  float acc[MT][NTO][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      m_run[mt][hf] = -INFINITY;
      lr[mt][hf] = lx[mt][hf] = 0.f;
    }
#pragma unroll
    for (int jn = 0; jn < NTO; ++jn)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][jn][e] = 0.f;
  }

  if (!__syncthreads_and(mbar_wait(smem_u32(&bar_q), 0, abort))) return;

  // One tile of keys: S = Q K^T for this warp's 16 keys, masked by `vis`,
  // online softmax update, P -> smem, O += P V for this warp's columns.
  const uint32_t sP = smem_u32(Ps);
  auto process = [&](uint32_t sK, uint32_t sV, auto vis) {
    float sc[MT][2][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[mt][j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        ldsm_x4(sw128_addr(sQ, 32, mt * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8), a[mt][0],
                a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t b0, b1;
        ldsm_x2(sw128_addr(sK, T, warp * 16 + j * 8 + (lane & 7), kk * 16 + ((lane >> 3) & 1) * 8),
                b0, b1);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          mma_16816(sc[mt][j], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
      }
    }
    // mask, scale, this warp's row maxima
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int key = warp * 16 + j * 8 + 2 * (lane & 3) + e2;
            float& x = sc[mt][j][hf * 2 + e2];
            x = vis(mt, hf, key) ? x * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if ((lane & 3) == 0) red[warp * 32 + mt * 16 + (lane >> 2) + hf * 8] = mx;
      }
    __syncthreads();
    // new running max, rescale of O and the sums, P
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int row = mt * 16 + (lane >> 2) + hf * 8;
        float mt_max = red[row];
#pragma unroll
        for (int w = 1; w < kSplitWarps; ++w) mt_max = fmaxf(mt_max, red[w * 32 + row]);
        const float m_new = fmaxf(m_run[mt][hf], mt_max);
        const float mb = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = ex2(m_run[mt][hf] - mb);  // exp2(-inf) = 0 on the first tile
        m_run[mt][hf] = m_new;
        lr[mt][hf] *= alpha;
        lx[mt][hf] *= alpha;
#pragma unroll
        for (int jn = 0; jn < NTO; ++jn) {
          acc[mt][jn][2 * hf] *= alpha;
          acc[mt][jn][2 * hf + 1] *= alpha;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float p0 = ex2(sc[mt][j][2 * hf] - mb);
          const float p1 = ex2(sc[mt][j][2 * hf + 1] - mb);
          const uint32_t pk = pack_bf16x2(p0, p1);
          lr[mt][hf] += bf16lo_to_f32(pk) + bf16hi_to_f32(pk);
          lx[mt][hf] += p0 + p1;
          const int col = warp * 16 + j * 8 + 2 * (lane & 3);
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + (row * LDP + col) * 2), "r"(pk)
                       : "memory");
        }
      }
    __syncthreads();
    // O += P V over the tile's 64 keys: this warp's head-dim columns
#pragma unroll
    for (int kk = 0; kk < T / 16; ++kk) {
      uint32_t a[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
        ldsm_x4(sP + ((mt * 16 + (lane & 15)) * LDP + kk * 16 + (lane >> 4) * 8) * 2, a[mt][0],
                a[mt][1], a[mt][2], a[mt][3]);
      const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int jp = 0; jp < NTO / 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sw128_addr(sV, T, key, warp * DW + jp * 16 + (lane >> 4) * 8), b0, b1, b2, b3);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          mma_16816(acc[mt][2 * jp], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
          mma_16816(acc[mt][2 * jp + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
        }
      }
    }
  };

  // ---- the tiles: cached positions, then (last range) the new tokens ---------
  for (int i = 0; i < nall; ++i) {
    const int st = i % kSplitStages;
    if (!__syncthreads_and(mbar_wait(smem_u32(&full[st]), (i / kSplitStages) & 1, abort))) return;
    const uint32_t sK = sKs + st * 2 * TILE, sV = sK + TILE;
    // V rows no key of this tile may use can hold anything (slots not written
    // yet, stale or never-initialised shared memory): zeroed, since P is 0
    // there and 0 * V must stay 0
    const int tp0 = t0 + i * T;  // position of key 0 of a cached tile
    const int first = i < ntile ? max(0, min(T, r1 - tp0)) : n_q;
    for (int idx = tid; idx < NCH * (T - first) * 8; idx += kSplitWarps * 32) {
      const int ch = idx / ((T - first) * 8);
      const int rem = idx - ch * (T - first) * 8;
      st_shared_zero16(sV + ch * T * 128 + (first + (rem >> 3)) * 128 + (rem & 7) * 16);
    }
    if (i < ntile) {
      process(sK, sV, [&](int mt, int hf, int key) {
        const int pk = tp0 + key;
        return pk >= vlo[mt][hf] && pk < r1;
      });
    } else {
      process(sK, sV, [&](int mt, int hf, int key) { return key < n_q && key <= trow[mt][hf]; });
    }
    __syncthreads();  // every warp is done with the stage and with P
    if (tid == 0 && i + kSplitStages < nall) {
      fence_proxy_async_smem();
      issue_tile(i + kSplitStages);
    }
  }

  // ---- partial state: row sums over the quad and the warps, then O, m, l ------
  float* outp = p.part + static_cast<size_t>(unit) * 32 * (D + 4);
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v = lr[mt][hf], x = lx[mt][hf];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      lr[mt][hf] = v;
      lx[mt][hf] = x;
    }
  // the sums of each warp cover its 16 keys of every tile: add over the warps
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        if ((lane & 3) == 0)
          red[warp * 32 + mt * 16 + (lane >> 2) + hf * 8] = pass == 0 ? lr[mt][hf] : lx[mt][hf];
    __syncthreads();
    if (tid < RP) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kSplitWarps; ++w) tot += red[w * 32 + tid];
      outp[tid * (D + 4) + D + 1 + pass] = tot;
    }
    __syncthreads();
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = mt * 16 + (lane >> 2) + hf * 8;
      float* orow = outp + row * (D + 4);
      if (warp == 0 && (lane & 3) == 0) orow[D] = m_run[mt][hf];
#pragma unroll
      for (int jn = 0; jn < NTO; ++jn) {
        const int col = warp * DW + jn * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(orow + col) =
            make_float2(acc[mt][jn][2 * hf], acc[mt][jn][2 * hf + 1]);
      }
    }
}

// Merge of the S partial states: one warp per (sequence, kv head, query row).
// Lanes take the ranges for the max and the sums, then every lane adds 4
// head-dim columns of each range's O (independent 16-byte loads).
template <int D>
__global__ void __launch_bounds__(32)
    decode_split_combine_kernel(const SplitParams p) {
  const int lane = threadIdx.x;
  const int bg = blockIdx.x / p.R, row = blockIdx.x - bg * p.R;
  const int b = bg / p.Hkv, g = bg - b * p.Hkv;
  const int t = row / p.G, hh = row - t * p.G;
  const int h = g * p.G + hh;
  const float* part = p.part + static_cast<size_t>(bg) * p.S * 32 * (D + 4);
  const float sk = p.sink != nullptr ? __ldg(p.sink + h) * kLog2e : -INFINITY;
  float M = sk;
  for (int r = lane; r < p.S; r += 32) M = fmaxf(M, part[(r * 32 + row) * (D + 4) + D]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float mb = (M == -INFINITY) ? 0.f : M;
  float L = 0.f, LX = 0.f;
  for (int r = lane; r < p.S; r += 32) {
    const float* pr = part + (r * 32 + row) * (D + 4);
    const float w = ex2(pr[D] - mb);  // an empty range has m = -inf: weight 0
    L += w * pr[D + 1];
    LX += w * pr[D + 2];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    L += __shfl_xor_sync(0xffffffffu, L, off);
    LX += __shfl_xor_sync(0xffffffffu, LX, off);
  }
  if (sk != -INFINITY) {
    const float ts = ex2(sk - mb);
    L += ts;
    LX += ts;
  }
  // O: lane takes columns [4 lane, 4 lane + 4) (D / 4 lanes)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane * 4 < D) {
    for (int r = 0; r < p.S; ++r) {
      const float* pr = part + (r * 32 + row) * (D + 4);
      const float w = ex2(__ldg(pr + D) - mb);
      const float4 v = __ldg(reinterpret_cast<const float4*>(pr) + lane);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const size_t orow = (static_cast<size_t>(b) * p.n_q + t) * p.Hq + h;
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(p.o + orow * D + lane * 4) = pk;
    if (lane == 0 && p.lse != nullptr) p.lse[orow] = (mb + lg2(LX)) * kLn2;
  }
}

}  // namespace swa
