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
// Three kernels, mma.sync m16n8k16 (bf16 in, fp32 accumulate) on
// shared-memory tiles (rows padded by 16 bytes: ldmatrix without bank
// conflicts):
//   bwd_prep_kernel  Delta from o and dO (fp32, [Hq, total] in the caller's
//                    workspace; coalesced 16-byte loads of whole rows) and
//                    dsink (per-CTA sums in shared memory, then atomic adds
//                    into the zeroed output)
//   bwd_dq_kernel    one CTA of 4 warps per (64 query rows = 64/G tokens x G
//                    heads, kv head): key blocks of 32 over the rows' window,
//                    double-buffered with cp.async; per warp 16 rows: S and
//                    dP (16 x 32), dS, dq += dS K
//   bwd_dkdv_kernel  one CTA of 8 warps per (128 keys, kv head): the query
//                    rows that see them in chunks of 32 (tokens x G heads),
//                    three buffers filled by cp.async (one barrier per
//                    chunk); per warp 16 keys: S^T
//                    and dP^T (16 x 32), dv += P^T dO, dk += dS^T q
// No inter-CTA waits; no traps.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_sm100.cuh"
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
  float* dsink;       // [Hq] or NULL; zero before bwd_prep_kernel
};

constexpr int kBwdPrepTokens = 16;  // tokens per prep CTA
constexpr int kBwdQRows = 64;      // query rows per dq CTA
constexpr int kBwdKeyBlock = 32;   // keys per dq step
constexpr int kBwdKeys = 128;      // keys per dk/dv CTA (8 warps x 16)
constexpr int kBwdRowChunk = 32;   // query rows per dk/dv step

__host__ __device__ inline size_t bwd_dq_smem_bytes(int D) {
  return static_cast<size_t>(2 * kBwdQRows + 4 * kBwdKeyBlock) * (D + 8) * 2;
}
__host__ __device__ inline size_t bwd_dkdv_smem_bytes(int D) {
  return static_cast<size_t>(2 * kBwdKeys + 6 * kBwdRowChunk) * (D + 8) * 2 +
         3 * 4 * kBwdRowChunk * sizeof(float);
}

// First key visible to token t (same sequence, inside the window), and the
// end of t's sequence.
__device__ __forceinline__ void bwd_token_bounds(const BwdParams& p, int t, int& first, int& end) {
  const int s = seq_of_token(p.cu_seqlens, p.num_seqs, t);
  const int lo = __ldg(p.cu_seqlens + s);
  end = __ldg(p.cu_seqlens + s + 1);
  first = p.window > 0 ? max(lo, t - p.window + 1) : lo;
}

// Copy `rows` rows of D bf16 (16-byte pieces) into a padded shared tile;
// src_row(r) gives the source row pointer or nullptr for a zero row.
template <int D, typename F>
__device__ __forceinline__ void bwd_load_rows(__nv_bfloat16* dst, int rows, F src_row) {
  constexpr int U = D / 8;  // 16-byte pieces per row
  for (int idx = threadIdx.x; idx < rows * U; idx += blockDim.x) {
    const int r = idx / U, u = idx - r * U;
    const __nv_bfloat16* s = src_row(r);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (s != nullptr) val = __ldg(reinterpret_cast<const uint4*>(s) + u);
    *reinterpret_cast<uint4*>(dst + r * (D + 8) + u * 8) = val;
  }
}

__device__ __forceinline__ uint32_t bwd_smem_addr(const __nv_bfloat16* base, int row, int col,
                                                  int ld) {
  return smem_u32(base + row * ld + col);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- Delta and dsink ------------------------------------------------------------
// Rows (token, head) are contiguous in o and dO: D/8 lanes take one row in
// 16-byte pieces (coalesced), four rows per group in flight; dsink partials
// gather per head in shared memory, one atomic add per head per CTA.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp per step
  constexpr int RPS = 8 * RPW;        // rows per CTA per step
  constexpr int UNR = 4;              // steps in flight
  extern __shared__ float prep_sink[];  // [Hq]
  const int tid = threadIdx.x, lane = tid & 31;
  const int sub = lane / LPR, pl = lane - sub * LPR;
  const long long row0 = static_cast<long long>(blockIdx.x) * kBwdPrepTokens * p.Hq;
  const long long row_end =
      min(row0 + static_cast<long long>(kBwdPrepTokens) * p.Hq,
          static_cast<long long>(p.total) * p.Hq);
  for (int h = tid; h < p.Hq; h += blockDim.x) prep_sink[h] = 0.f;
  __syncthreads();
  const long long my0 = row0 + (tid >> 5) * RPW + sub;
  for (long long base = my0; base < row_end; base += static_cast<long long>(RPS) * UNR) {
    uint4 a[UNR], b[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const long long row = base + static_cast<long long>(u) * RPS;
      a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
      if (row < row_end) {
        a[u] = __ldg(reinterpret_cast<const uint4*>(p.o + row * D) + pl);
        b[u] = __ldg(reinterpret_cast<const uint4*>(p.dout + row * D) + pl);
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
      const uint32_t bv[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        acc += bf16lo_to_f32(av[e]) * bf16lo_to_f32(bv[e]) +
               bf16hi_to_f32(av[e]) * bf16hi_to_f32(bv[e]);
#pragma unroll
      for (int m = LPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
      const long long row = base + static_cast<long long>(u) * RPS;
      if (pl == 0 && row < row_end) {
        const int t = static_cast<int>(row / p.Hq), h = static_cast<int>(row - t * p.Hq);
        const size_t li = static_cast<size_t>(h) * p.total + t;
        p.delta[li] = acc;
        if (p.sink != nullptr)
          atomicAdd(&prep_sink[h], -expf(__ldg(p.sink + h) - __ldg(p.lse + li)) * acc);
      }
    }
  }
  __syncthreads();
  if (p.dsink != nullptr && p.sink != nullptr)
    for (int h = tid; h < p.Hq; h += blockDim.x) atomicAdd(p.dsink + h, prep_sink[h]);
}

// ---- dq -------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) bwd_dq_kernel(const BwdParams p) {
  constexpr int LD = D + 8;
  constexpr int NTD = D / 8;  // n8 tiles over the head dim
  constexpr int U = D / 8;    // 16-byte pieces per row
  constexpr int KB = kBwdKeyBlock;
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(bwd_smem);
  __nv_bfloat16* sdO = sQ + kBwdQRows * LD;
  __nv_bfloat16* sKb = sdO + kBwdQRows * LD;  // [2][KB][LD]
  __nv_bfloat16* sVb = sKb + 2 * KB * LD;     // [2][KB][LD]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int TQ = kBwdQRows / p.G;  // tokens per CTA
  const int n_tiles = (p.total + TQ - 1) / TQ;
  // the last query tiles (the most keys, in a global layer) first, all kv
  // heads of a tile together
  const int g = blockIdx.x % p.Hkv;
  const int t0 = (n_tiles - 1 - static_cast<int>(blockIdx.x) / p.Hkv) * TQ;

  // the Q and dO rows of the tile (first cp.async group, with key block 0)
  for (int idx = tid; idx < kBwdQRows * U * 2; idx += blockDim.x) {
    const int which = idx / (kBwdQRows * U);
    const int rem = idx - which * kBwdQRows * U;
    const int r = rem / U, u = rem - r * U;
    const int t = t0 + r / p.G;
    const bool ok = t < p.total;
    const __nv_bfloat16* src = (which == 0 ? p.q : p.dout) +
                               (static_cast<size_t>(ok ? t : t0) * p.Hq + g * p.G + r % p.G) * D +
                               u * 8;
    cp_async16(smem_u32((which == 0 ? sQ : sdO) + r * LD + u * 8), src, ok);
  }
  // keys: from the first token's first visible key to the last token
  int kmin, kend;
  bwd_token_bounds(p, t0, kmin, kend);
  const int kmax = min(t0 + TQ, p.total) - 1;
  const int n_blocks = (kmax - kmin) / KB + 1;
  auto load_block = [&](int bl) {
    const int j0 = kmin + bl * KB, bf = bl & 1;
    for (int idx = tid; idx < KB * U * 2; idx += blockDim.x) {
      const int which = idx / (KB * U);
      const int rem = idx - which * KB * U;
      const int r = rem / U, u = rem - r * U;
      const int j = j0 + r;
      const bool ok = j <= kmax;
      const __nv_bfloat16* src =
          (which == 0 ? p.k : p.v) + (static_cast<size_t>(ok ? j : kmin) * p.Hkv + g) * D + u * 8;
      cp_async16(smem_u32((which == 0 ? sKb : sVb) + (bf * KB + r) * LD + u * 8), src, ok);
    }
  };
  load_block(0);
  cp_async_commit();

  // this thread's two rows (fragment rows lane/4 and lane/4 + 8 of its warp)
  int tok[2], first[2];
  float lse2[2], dlt[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int r = warp * 16 + (lane >> 2) + hf * 8;
    const int t = t0 + r / p.G;
    tok[hf] = t < p.total ? t : -1;
    first[hf] = 0x7fffffff;
    lse2[hf] = 0.f;
    dlt[hf] = 0.f;
    if (t < p.total) {
      int end;
      bwd_token_bounds(p, t, first[hf], end);
      const size_t li = static_cast<size_t>(g * p.G + r % p.G) * p.total + t;
      lse2[hf] = __ldg(p.lse + li) * kLog2e;
      dlt[hf] = p.delta[li];
    }
  }
  // the key range of this warp's rows (warp-uniform): blocks outside it are
  // skipped
  int fmin = min(first[0], first[1]), tmax = max(tok[0], tok[1]);
#pragma unroll
  for (int m = 4; m < 32; m <<= 1) {
    fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, m));
    tmax = max(tmax, __shfl_xor_sync(0xffffffffu, tmax, m));
  }

  float acc[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;

  for (int bl = 0; bl < n_blocks; ++bl) {
    if (bl + 1 < n_blocks) {
      load_block(bl + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // block bl (and, first time, the Q / dO rows) landed
    const int j0 = kmin + bl * KB;
    const __nv_bfloat16* sK = sKb + (bl & 1) * KB * LD;
    const __nv_bfloat16* sV = sVb + (bl & 1) * KB * LD;
    if (!(tmax < j0 || fmin > j0 + KB - 1)) {
      // S = Q K^T and dP = dO V^T for this warp's 16 rows x 32 keys
      float s[4][4], dp[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4], ao[4];
        const int arow = warp * 16 + (lane & 15), acol = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(bwd_smem_addr(sQ, arow, acol, LD), a[0], a[1], a[2], a[3]);
        ldsm_x4(bwd_smem_addr(sdO, arow, acol, LD), ao[0], ao[1], ao[2], ao[3]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const int brow = np * 16 + (lane & 7) + (lane >> 4) * 8;
          const int bcol = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(bwd_smem_addr(sK, brow, bcol, LD), b0, b1, b2, b3);
          mma_16816(s[2 * np], a[0], a[1], a[2], a[3], b0, b1);
          mma_16816(s[2 * np + 1], a[0], a[1], a[2], a[3], b2, b3);
          ldsm_x4(bwd_smem_addr(sV, brow, bcol, LD), b0, b1, b2, b3);
          mma_16816(dp[2 * np], ao[0], ao[1], ao[2], ao[3], b0, b1);
          mma_16816(dp[2 * np + 1], ao[0], ao[1], ao[2], ao[3], b2, b3);
        }
      }
      // dS = P (dP - Delta), P recomputed from the forward's lse; 0 off the mask
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hf = e >> 1;
          const int j = j0 + n * 8 + 2 * (lane & 3) + (e & 1);
          const bool vis = tok[hf] >= 0 && j >= first[hf] && j <= tok[hf];
          const float pr = vis ? ex2(fmaf(s[n][e], p.scale_log2, -lse2[hf])) : 0.f;
          s[n][e] = pr * (dp[n][e] - dlt[hf]);
        }
      // dq += dS K over the block's 32 keys (two k16 steps)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const uint32_t a0 = pack_bf16x2(s[2 * ks][0], s[2 * ks][1]);
        const uint32_t a1 = pack_bf16x2(s[2 * ks][2], s[2 * ks][3]);
        const uint32_t a2 = pack_bf16x2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
        const uint32_t a3 = pack_bf16x2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
        for (int np = 0; np < NTD / 2; ++np) {
          const int krow = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int kcol = np * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(bwd_smem_addr(sK, krow, kcol, LD), b0, b1, b2, b3);
          mma_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
          mma_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncthreads();  // buffer bl & 1 is read: the load two blocks on may overwrite it
  }
  // dq = scale * acc -> bf16
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (tok[hf] < 0) continue;
    const int r = warp * 16 + (lane >> 2) + hf * 8;
    __nv_bfloat16* dst = p.dq + (static_cast<size_t>(tok[hf]) * p.Hq + g * p.G + r % p.G) * D;
#pragma unroll
    for (int n = 0; n < NTD; ++n)
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * (lane & 3)) =
          pack_bf16x2(acc[n][2 * hf] * p.scale, acc[n][2 * hf + 1] * p.scale);
  }
}

// ---- dk, dv ---------------------------------------------------------------------
// One CTA of 8 warps per (128 keys, kv head); warp w owns keys 16w .. 16w+15
// and accumulates their dk and dv (16 x D each) in registers. The rows that
// see the keys come in chunks of 32 (tokens x G heads), double-buffered with
// cp.async: the next chunk's q and dO rows land while this one is computed.
template <int D>
__global__ void __launch_bounds__(256, 1) bwd_dkdv_kernel(const BwdParams p) {
  constexpr int LD = D + 8;
  constexpr int NTD = D / 8;
  constexpr int KT = kBwdKeys, RC = kBwdRowChunk;
  constexpr int U = D / 8;  // 16-byte pieces per row
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(bwd_smem);
  __nv_bfloat16* sV = sK + KT * LD;
  __nv_bfloat16* sQb = sV + KT * LD;     // [3][RC][LD]
  __nv_bfloat16* sdOb = sQb + 3 * RC * LD;  // [3][RC][LD]
  float* rlse2b = reinterpret_cast<float*>(sdOb + 3 * RC * LD);  // [3][RC] lse (natural log)
  float* rdltb = rlse2b + 3 * RC;
  int* rtokb = reinterpret_cast<int*>(rdltb + 3 * RC);
  int* rfirstb = rtokb + 3 * RC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the first key tiles (the most rows, in a global layer) first, all kv
  // heads of a tile together
  const int g = blockIdx.x % p.Hkv;
  const int k0 = (static_cast<int>(blockIdx.x) / p.Hkv) * KT;
  const int klast = min(k0 + KT, p.total) - 1;

  // rows that see any of these keys: tokens k0 .. the last one that sees klast
  int f_unused, end_last;
  bwd_token_bounds(p, klast, f_unused, end_last);
  const int i_hi = p.window > 0 ? min(klast + p.window - 1, end_last - 1) : end_last - 1;
  const int n_rows = (i_hi - k0 + 1) * p.G;
  const int n_chunks = (n_rows + RC - 1) / RC;
  int c_lo = 0, c_hi = -1;  // sequence of the last row token looked up

  // chunk c of the rows into buffer c % 3 (q, dO, lse and Delta by cp.async;
  // token and first key by plain stores)
  auto prefetch = [&](int c) {
    const int bf = c % 3;
    for (int idx = tid; idx < RC * U * 2; idx += blockDim.x) {
      const int which = idx / (RC * U);  // 0: q, 1: dO
      const int rem = idx - which * RC * U;
      const int r = rem / U, u = rem - r * U;
      const int rr = c * RC + r;
      const bool ok = rr < n_rows;
      const int t = k0 + (ok ? rr / p.G : 0);
      const __nv_bfloat16* src = (which == 0 ? p.q : p.dout) +
                                 (static_cast<size_t>(t) * p.Hq + g * p.G + (ok ? rr % p.G : 0)) * D +
                                 u * 8;
      __nv_bfloat16* dst = (which == 0 ? sQb : sdOb) + (bf * RC + r) * LD + u * 8;
      cp_async16(smem_u32(dst), src, ok);
    }
    if (tid < RC) {
      // the row's token and first key (sequence bounds cached across chunks:
      // tokens only grow), its lse and Delta by cp.async like the rows
      const int rr = c * RC + tid;
      const bool ok = rr < n_rows;
      int t = -1, first = 0x7fffffff;
      size_t li = 0;
      if (ok) {
        t = k0 + rr / p.G;
        if (t >= c_hi) {
          const int sq = seq_of_token(p.cu_seqlens, p.num_seqs, t);
          c_lo = __ldg(p.cu_seqlens + sq);
          c_hi = __ldg(p.cu_seqlens + sq + 1);
        }
        first = p.window > 0 ? max(c_lo, t - p.window + 1) : c_lo;
        li = static_cast<size_t>(g * p.G + rr % p.G) * p.total + t;
      }
      rtokb[bf * RC + tid] = t;
      rfirstb[bf * RC + tid] = first;
      cp_async4(smem_u32(rlse2b + bf * RC + tid), p.lse + li, ok);
      cp_async4(smem_u32(rdltb + bf * RC + tid), p.delta + li, ok);
    }
  };

  // K and V of the tile (part of the first group)
  for (int idx = tid; idx < KT * U * 2; idx += blockDim.x) {
    const int which = idx / (KT * U);
    const int rem = idx - which * KT * U;
    const int r = rem / U, u = rem - r * U;
    const int j = k0 + r;
    const bool ok = j <= klast;
    const __nv_bfloat16* src =
        (which == 0 ? p.k : p.v) + (static_cast<size_t>(ok ? j : k0) * p.Hkv + g) * D + u * 8;
    cp_async16(smem_u32((which == 0 ? sK : sV) + r * LD + u * 8), src, ok);
  }
  prefetch(0);
  cp_async_commit();

  int key[2];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) key[hf] = k0 + warp * 16 + (lane >> 2) + hf * 8;

  float dk[NTD][4], dv[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

  for (int c = 0; c < n_chunks; ++c) {
    if (c + 1 < n_chunks) {
      prefetch(c + 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    // chunk c (and K, V) landed and its row data are visible; and every
    // thread is past chunk c - 1, so the prefetch of chunk c + 2 (next
    // iteration) may overwrite buffer (c - 1) % 3 -- one barrier per chunk
    __syncthreads();
    const int bf = c % 3;
    const __nv_bfloat16* sQ = sQb + bf * RC * LD;
    const __nv_bfloat16* sdO = sdOb + bf * RC * LD;
    const float* rlse2 = rlse2b + bf * RC;
    const float* rdlt = rdltb + bf * RC;
    const int* rtok = rtokb + bf * RC;
    const int* rfirst = rfirstb + bf * RC;
    // a block wholly off the band (every row of the chunk sees none of this
    // warp's keys) adds nothing: the warp skips its MMAs (the decision is the
    // same for the whole warp: it depends on the chunk's tokens and the
    // warp's keys only)
    {
      const int t_first = rtok[0];
      const int t_last = rtok[RC - 1] >= 0 ? rtok[RC - 1] : p.total - 1;
      const int kw0 = k0 + warp * 16, kw1 = min(kw0 + 15, klast);
      const bool none = kw0 > klast || t_last < kw0 ||
                        (p.window > 0 && t_first > kw1 + p.window - 1);
      if (none) continue;
    }
    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 32 rows
    float s[4][4], dp[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], av[4];
      const int arow = warp * 16 + (lane & 15), acol = kk * 16 + (lane >> 4) * 8;
      ldsm_x4(bwd_smem_addr(sK, arow, acol, LD), a[0], a[1], a[2], a[3]);
      ldsm_x4(bwd_smem_addr(sV, arow, acol, LD), av[0], av[1], av[2], av[3]);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int brow = np * 16 + (lane & 7) + (lane >> 4) * 8;
        const int bcol = kk * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(bwd_smem_addr(sQ, brow, bcol, LD), b0, b1, b2, b3);
        mma_16816(s[2 * np], a[0], a[1], a[2], a[3], b0, b1);
        mma_16816(s[2 * np + 1], a[0], a[1], a[2], a[3], b2, b3);
        ldsm_x4(bwd_smem_addr(sdO, brow, bcol, LD), b0, b1, b2, b3);
        mma_16816(dp[2 * np], av[0], av[1], av[2], av[3], b0, b1);
        mma_16816(dp[2 * np + 1], av[0], av[1], av[2], av[3], b2, b3);
      }
    }
    // P^T and dS^T; 0 off the mask
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rr = n * 8 + 2 * (lane & 3) + (e & 1);
        const int j = key[e >> 1];
        const int t = rtok[rr];
        const bool vis = t >= 0 && j <= klast && j >= rfirst[rr] && j <= t;
        const float pr = vis ? ex2(fmaf(s[n][e], p.scale_log2, -rlse2[rr] * kLog2e)) : 0.f;
        s[n][e] = pr;
        dp[n][e] = pr * (dp[n][e] - rdlt[rr]);
      }
    // dv += P^T dO and dk += dS^T Q over the chunk's 32 rows (two k16 steps)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t pa0 = pack_bf16x2(s[2 * ks][0], s[2 * ks][1]);
      const uint32_t pa1 = pack_bf16x2(s[2 * ks][2], s[2 * ks][3]);
      const uint32_t pa2 = pack_bf16x2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
      const uint32_t pa3 = pack_bf16x2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
      const uint32_t da0 = pack_bf16x2(dp[2 * ks][0], dp[2 * ks][1]);
      const uint32_t da1 = pack_bf16x2(dp[2 * ks][2], dp[2 * ks][3]);
      const uint32_t da2 = pack_bf16x2(dp[2 * ks + 1][0], dp[2 * ks + 1][1]);
      const uint32_t da3 = pack_bf16x2(dp[2 * ks + 1][2], dp[2 * ks + 1][3]);
#pragma unroll
      for (int np = 0; np < NTD / 2; ++np) {
        const int brow = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int bcol = np * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(bwd_smem_addr(sdO, brow, bcol, LD), b0, b1, b2, b3);
        mma_16816(dv[2 * np], pa0, pa1, pa2, pa3, b0, b1);
        mma_16816(dv[2 * np + 1], pa0, pa1, pa2, pa3, b2, b3);
        ldsm_x4_t(bwd_smem_addr(sQ, brow, bcol, LD), b0, b1, b2, b3);
        mma_16816(dk[2 * np], da0, da1, da2, da3, b0, b1);
        mma_16816(dk[2 * np + 1], da0, da1, da2, da3, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  // dk = scale * acc, dv -> bf16
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    const int j = key[hf];
    if (j > klast) continue;
    __nv_bfloat16* dkr = p.dk + (static_cast<size_t>(j) * p.Hkv + g) * D;
    __nv_bfloat16* dvr = p.dv + (static_cast<size_t>(j) * p.Hkv + g) * D;
#pragma unroll
    for (int n = 0; n < NTD; ++n) {
      const int c = n * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(dkr + c) =
          pack_bf16x2(dk[n][2 * hf] * p.scale, dk[n][2 * hf + 1] * p.scale);
      *reinterpret_cast<uint32_t*>(dvr + c) = pack_bf16x2(dv[n][2 * hf], dv[n][2 * hf + 1]);
    }
  }
}

}  // namespace swa
