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
// are cut into S ranges of `chunk` positions (a multiple of kSplitTile). The
// tcgen05 kernel of decode_splitkv_tc_sm100.cuh streams each range and writes
// its partial state (max in log2 units, unnormalised O, two row sums); the
// last range also takes the n_q new tokens. The merge kernel below combines
// the S partial states of each row and adds the sink term once:
//   M = max(s, max_r m_r),  O = sum_r 2^(m_r - M) O_r / L,
//   L = sum_r 2^(m_r - M) l_r + 2^(s - M),  LSE = (M + log2(same with l_x)) ln 2.
// A range with m = -inf (no position, no new token) is skipped: its sums and
// O may be left unwritten.
//
// Every wait is bounded (see mbar_wait); nothing here traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "decode_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kSplitTile = 64;    // cached positions per tile of the cache

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
  // an empty range has m = -inf (weight 0) and may leave its sums and O
  // unwritten: it is skipped
  float L = 0.f, LX = 0.f;
  for (int r = lane; r < p.S; r += 32) {
    const float* pr = part + (r * 32 + row) * (D + 4);
    if (pr[D] == -INFINITY) continue;
    const float w = ex2(pr[D] - mb);
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
      const float m = __ldg(pr + D);
      if (m == -INFINITY) continue;
      const float w = ex2(m - mb);
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
