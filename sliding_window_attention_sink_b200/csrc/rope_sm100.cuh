// rope_sm100.cuh -- rotary position embedding for the prefill: the rotation of
// one 8-pair group of a bf16 row (used in shared memory by the fused ring
// prefill), the angle arithmetic, and a standalone pass that rotates q and k
// into a workspace for the prefill kernels that do not rotate in place.
//
// Operation. The MiMo-V2-Flash report summary (mlpod.com), section 3.1 "Data
// Scheduler", gives the RoPE base per layer type (SWA 10,000; global 640,000,
// then 5,000,000); the ICML talk write-up (hzrcw.cc), Q&A on position
// encoding, says positions keep increasing while the window slides. The
// rotation is the standard rotary embedding over the whole head dimension:
// pair c (c < D/2) turns by p * theta_c, theta_c = base^(-2c/D), at absolute
// position p; the pair is (c, c + D/2) ("rotate half") or (2c, 2c + 1)
// (interleaved). Rotated values are rounded to bf16 (they feed bf16 MMAs and
// the bf16 ring).
//
// Angles. theta_c / (2 pi) is passed as two floats (hi + lo, from a double on
// the host); p < 2^24 is exact in float, p * hi is split exactly with an FMA,
// its integer part dropped exactly, and sin / cos of the remaining fraction of
// a turn come from sincospif. The angle error is a few 1e-8 rad at any
// position below 2^24, so the rotated values are the correctly rounded bf16
// of the exact rotation except within about 1e-7 relative of a rounding
// boundary.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "prefill_sm100.cuh"
#include "ptx_sm100.cuh"

namespace swa {

constexpr int kRopeMaxPairs = 64;      // D / 2 for D = 128
constexpr int kRopeMaxPos = 1 << 24;   // positions are exact in float below this

struct RopeArgs {
  const int32_t* pos0;   // [num_seqs] first position of each sequence, or NULL (0)
  int interleaved;       // 0: pairs (c, c + D/2); 1: pairs (2c, 2c + 1)
  float f_hi[kRopeMaxPairs], f_lo[kRopeMaxPairs];  // theta_c / (2 pi) = hi + lo
  __nv_bfloat16* k_ring;  // [num_seqs, ring_W, Hkv, D] or NULL: no ring written
  __nv_bfloat16* v_ring;
  int ring_W;
};

// cos and sin of p * theta_c for the 8 pairs c = c0 .. c0 + 7.
__device__ __forceinline__ void rope_cos_sin8(const RopeArgs& r, int p, int c0, float (&cs)[8],
                                              float (&sn)[8]) {
  const float pf = static_cast<float>(p);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float hi = r.f_hi[c0 + e], lo = r.f_lo[c0 + e];
    const float th = pf * hi;
    const float te = fmaf(pf, hi, -th);  // p * hi = th + te exactly
    const float fr = th - rintf(th);     // exact: |fr| <= 1/2
    const float t = fr + fmaf(pf, lo, te);
    sincospif(2.0f * t, &sn[e], &cs[e]);
  }
}

// Rotate the 8 pairs held in two 16-byte units a (4 bf16x2) and b: rotate
// half pairs a[e] with b[e]; interleaved, the pairs are adjacent elements
// (4 in a, then 4 in b). cs / sn are the 8 pairs' cos / sin in that order.
__device__ __forceinline__ void rope_rotate8(uint32_t (&a)[4], uint32_t (&b)[4],
                                             const float (&cs)[8], const float (&sn)[8],
                                             bool interleaved) {
  if (!interleaved) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x0 = bf16lo_to_f32(a[i]), x1 = bf16hi_to_f32(a[i]);
      const float y0 = bf16lo_to_f32(b[i]), y1 = bf16hi_to_f32(b[i]);
      const int e = 2 * i;
      a[i] = pack_bf16x2(fmaf(x0, cs[e], -y0 * sn[e]), fmaf(x1, cs[e + 1], -y1 * sn[e + 1]));
      b[i] = pack_bf16x2(fmaf(y0, cs[e], x0 * sn[e]), fmaf(y1, cs[e + 1], x1 * sn[e + 1]));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float x = bf16lo_to_f32(a[i]), y = bf16hi_to_f32(a[i]);
      a[i] = pack_bf16x2(fmaf(x, cs[i], -y * sn[i]), fmaf(y, cs[i], x * sn[i]));
      const float u = bf16lo_to_f32(b[i]), w = bf16hi_to_f32(b[i]);
      b[i] = pack_bf16x2(fmaf(u, cs[4 + i], -w * sn[4 + i]), fmaf(w, cs[4 + i], u * sn[4 + i]));
    }
  }
}

// Head-dim offsets (elements) of the two 16-byte units of 8-pair group k
// (0 <= k < D/16).
template <int D>
__device__ __forceinline__ void rope_units(int k, bool interleaved, int& da, int& db) {
  if (interleaved) {
    da = 16 * k;
    db = 16 * k + 8;
  } else {
    da = 8 * k;
    db = D / 2 + 8 * k;
  }
}

// Absolute position of packed token t (0 <= t < total): pos0[s] + (t - cu[s]).
// The caller keeps the bounds [s_lo, s_hi), index s and first position p0 of
// the last sequence looked up (start with s_lo > s_hi). Positions outside
// [0, 2^24) are flagged (bit 1) and clamped.
__device__ __forceinline__ int rope_token_pos(const int32_t* cu, int num_seqs, const int32_t* pos0,
                                              int t, int& s_lo, int& s_hi, int& s, int& p0) {
  if (t < s_lo || t >= s_hi) {
    s = seq_of_token(cu, num_seqs, t);
    s_lo = __ldg(cu + s);
    s_hi = __ldg(cu + s + 1);
    p0 = pos0 != nullptr ? __ldg(pos0 + s) : 0;
  }
  long long p = static_cast<long long>(p0) + (t - s_lo);
  if (p < 0 || p >= kRopeMaxPos) {
    flag_error(2u);
    p = p < 0 ? 0 : kRopeMaxPos - 1;
  }
  return static_cast<int>(p);
}

// 16-byte global store / load.
__device__ __forceinline__ void st_global_v4(void* ptr, const uint32_t (&v)[4]) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void ld_global_v4(const void* ptr, uint32_t (&v)[4]) {
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "l"(ptr));
}

// Standalone pass (for the prefill kernels that read q and k through TMA
// without rotating them): one CTA per packed token rotates its Hq query rows
// and Hkv key rows into q_out / k_out, and, for the last ring_W tokens of each
// sequence, writes the rotated key row and the value row into the ring at
// slot (position mod ring_W).
struct RopePassParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_out;
  const int32_t* cu_seqlens;
  int num_seqs, total, Hq, Hkv;
};

template <int D>
__global__ void __launch_bounds__(128) rope_pass_kernel(const RopePassParams p, const RopeArgs r) {
  constexpr int NK = D / 16;  // 8-pair groups per row
  __shared__ float cs_sh[D / 2], sn_sh[D / 2];
  const int t = blockIdx.x;
  int s_lo = 1, s_hi = 0, s = 0, p0 = 0;
  const int pos = rope_token_pos(p.cu_seqlens, p.num_seqs, r.pos0, t, s_lo, s_hi, s, p0);
  if (threadIdx.x < NK) {
    float cs[8], sn[8];
    rope_cos_sin8(r, pos, 8 * threadIdx.x, cs, sn);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cs_sh[8 * threadIdx.x + e] = cs[e];
      sn_sh[8 * threadIdx.x + e] = sn[e];
    }
  }
  __syncthreads();
  const bool inter = r.interleaved != 0;
  const bool emit = r.k_ring != nullptr && t - s_lo >= (s_hi - s_lo) - r.ring_W;
  const size_t ring_row =
      (static_cast<size_t>(s) * r.ring_W + static_cast<size_t>(pos) % r.ring_W) * p.Hkv;
  const int n_items = (p.Hq + p.Hkv) * NK;
  for (int it = threadIdx.x; it < n_items; it += blockDim.x) {
    const int h = it / NK, k = it - h * NK;
    int da, db;
    rope_units<D>(k, inter, da, db);
    const bool is_q = h < p.Hq;
    const __nv_bfloat16* src =
        is_q ? p.q + (static_cast<size_t>(t) * p.Hq + h) * D
             : p.k + (static_cast<size_t>(t) * p.Hkv + (h - p.Hq)) * D;
    __nv_bfloat16* dst = is_q ? p.q_out + (static_cast<size_t>(t) * p.Hq + h) * D
                              : p.k_out + (static_cast<size_t>(t) * p.Hkv + (h - p.Hq)) * D;
    uint32_t a[4], b[4];
    ld_global_v4(src + da, a);
    ld_global_v4(src + db, b);
    float cs[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cs[e] = cs_sh[8 * k + e];
      sn[e] = sn_sh[8 * k + e];
    }
    rope_rotate8(a, b, cs, sn, inter);
    st_global_v4(dst + da, a);
    st_global_v4(dst + db, b);
    if (!is_q && emit) {
      const int g = h - p.Hq;
      __nv_bfloat16* kr = r.k_ring + (ring_row + g) * D;
      __nv_bfloat16* vr = r.v_ring + (ring_row + g) * D;
      st_global_v4(kr + da, a);
      st_global_v4(kr + db, b);
      const __nv_bfloat16* vs = p.v + (static_cast<size_t>(t) * p.Hkv + g) * D;
      ld_global_v4(vs + da, a);
      ld_global_v4(vs + db, b);
      st_global_v4(vr + da, a);
      st_global_v4(vr + db, b);
    }
  }
}

}  // namespace swa
