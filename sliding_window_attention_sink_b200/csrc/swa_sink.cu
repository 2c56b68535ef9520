// swa_sink.cu -- the C ABI of libswasink.so (declared in include/swa_sink.h):
// argument validation, TMA tensor-map encoding and kernel launches for the
// sliding-window / global attention with a per-head sink on sm_100a.
//
// The operation and its sources are described in include/swa_sink.h. Every
// argument error is returned before any launch. The library allocates no
// device memory; its only device-side state is the error-flag word and the
// eight static scheduler slots of swa_sink_attn_fwd_noalloc.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <mutex>
#include <utility>

#include "../../include/swa_sink.h"
#include "backward_sm100.cuh"
#include "decode_fp8_sm100.cuh"
#include "decode_sm100.cuh"
#include "decode_tc_sm100.cuh"
#include "decode_splitkv_sm100.cuh"
#include "decode_splitkv_tc_sm100.cuh"
#include "prefill_chunked_sm100.cuh"
#include "prefill_sm100.cuh"
#include "prefill_swa_ring_sm100.cuh"
#include "rope_sm100.cuh"

namespace {

constexpr int kMaxDevices = 64;

// ---- driver entry point for cuTensorMapEncodeTiled (no -lcuda needed) -------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int cuda_fail(const char* what, int err);

// 3-D bf16 tensor [outer][mid][inner] (inner contiguous), 128-byte swizzle.
int encode_3d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t mid,
              uint64_t outer, uint32_t box_inner, uint32_t box_mid, uint32_t box_outer) {
  auto fn = get_encode_fn();
  if (!fn) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0);
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {box_inner, box_mid, box_outer};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : cuda_fail("cuTensorMapEncodeTiled", static_cast<int>(r));
}

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 contiguous), 128-byte swizzle.
int encode_4d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  auto fn = get_encode_fn();
  if (!fn) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0);
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : cuda_fail("cuTensorMapEncodeTiled", static_cast<int>(r));
}

// 4-D byte tensor [d3][d2][d1][d0] (E4M3 codes, d0 contiguous), boxes of b0
// bytes inner: the 128-byte swizzle for 128-byte rows, the 64-byte one for
// 64-byte rows.
int encode_u8_4d(CUtensorMap* map, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  auto fn = get_encode_fn();
  if (!fn) return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0);
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0, d0 * d1, d0 * d1 * d2};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  b0 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SWA_OK : cuda_fail("cuTensorMapEncodeTiled", static_cast<int>(r));
}

// With SWA_SINK_DEBUG set in the environment, failing CUDA calls are named
// on stderr (the status code alone says only SWA_ERR_CUDA).
int cuda_fail(const char* what, int err) {
  static const bool debug = std::getenv("SWA_SINK_DEBUG") != nullptr;
  if (debug) std::fprintf(stderr, "swa_sink: %s failed (%d)\n", what, err);
  return SWA_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` (once per size
// increase, per device). The limit plus the kernel's static shared memory
// must stay within the device's opt-in maximum.
std::mutex g_attr_mu;
template <typename K>
int ensure_smem_attr(K kernel, size_t bytes, size_t (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (done[dev] < bytes) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bytes));
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
    done[dev] = bytes;
  }
  return SWA_OK;
}

// Prefer the largest shared-memory carve-out of the unified L1 / shared
// array for a kernel (once per device).
template <typename K>
int ensure_carveout(K kernel, bool (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_attr_mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             static_cast<int>(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(carveout)", e);
    done[dev] = true;
  }
  return SWA_OK;
}
bool g_carve_dec[2][2][2][kMaxDevices];

size_t g_attr_prefill64[kMaxDevices], g_attr_prefill128[kMaxDevices];
size_t g_attr_dec[2][2][2][2][kMaxDevices];
size_t g_attr_dec_tc[2][kMaxDevices];

int next_pow2(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

size_t g_attr_ring[2][2][swa::kRingMaxBN16 + 1][kMaxDevices];

// ---- scheduler slots that need no allocation ------------------------------------
// swa_sink_attn_fwd_noalloc runs the ring kernel with a software tile
// scheduler whose counters live in this static array. Each slot is two words
// that must read zero when a launch starts: they are zero when the module
// loads, and every launch leaves its slot zero again (its last CTA clears
// it). 8 slots = 64 bytes.
constexpr int kNoAllocSlots = 8;
static __device__ __align__(256) unsigned int g_noalloc_sched[2 * kNoAllocSlots];
std::mutex g_noalloc_mu;
unsigned int* g_noalloc_base[kMaxDevices];

int raise_prefill_smem_limits();

// The device address of the slot. The first call on a device (with that
// device current) looks the array up with cudaGetSymbolAddress and does the
// rest of the one-time set-up of every prefill kernel this call can run (the
// shared-memory limits, the tensor-map entry point), so later calls make no
// set-up call of any kind.
int noalloc_slot(int slot, unsigned int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cuda_fail("cudaGetDevice", e);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_base[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_sched);
    if (e != cudaSuccess || ptr == nullptr) return cuda_fail("cudaGetSymbolAddress", e);
    if (raise_prefill_smem_limits() != SWA_OK) return SWA_ERR_CUDA;
    if (get_encode_fn() == nullptr)
      return cuda_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0);
    g_noalloc_base[dev] = static_cast<unsigned int*>(ptr);
  }
  *out = g_noalloc_base[dev] + 2 * slot;
  return SWA_OK;
}

// Work units of the ring kernel over n_tiles tiles on nsm SMs: each of the
// first min(nsm, n_tiles) units is a static share of static_tiles consecutive
// tiles (about kStaticShare of an even split); the rest of the tiles go out in
// ranges of kRingDynSpan to whichever CTA is free, so SMs that run faster take
// more. (On B200 the same tile stream ran up to 1.3x faster on some SMs than
// on others.) A ring range refills the K/V window once (NWIN - 1 extra
// blocks). With no counter (counted == false) an empty static share is left
// out: the launch has one CTA per non-empty unit. Returns the number of units.
constexpr double kStaticShare = 0.75;
constexpr int kRingDynSpan = 8;
int ring_schedule(int n_tiles, int nsm, bool counted, swa::RingParams* p) {
  const int lead = std::min(nsm, n_tiles);
  p->static_tiles = static_cast<int>(kStaticShare * n_tiles / lead);
  p->n_static = (p->static_tiles > 0 || counted) ? lead : 0;
  p->dyn_base = p->static_tiles * p->n_static;
  p->dyn_span = kRingDynSpan;
  const long long n_dyn = (static_cast<long long>(n_tiles) - p->dyn_base + kRingDynSpan - 1) /
                          kRingDynSpan;
  return static_cast<int>(p->n_static + n_dyn);
}

template <int D, int BN16, bool ROPE>
int run_ring(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
             const CUtensorMap& to, const swa::RingParams& p, const swa::RopeArgs& rope,
             size_t smem, int grid, cudaStream_t st) {
  auto kern = swa::prefill_swa_ring_kernel<D, BN16, ROPE>;
  if (ensure_smem_attr(kern, smem, g_attr_ring[ROPE][D == 128][BN16]) != SWA_OK)
    return SWA_ERR_CUDA;
  kern<<<grid, swa::kRingThreads, smem, st>>>(tq, tk, tv, to, p, rope);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("ring prefill launch", e);
}

// Dynamic shared memory available next to the ring kernel's static barriers.
constexpr size_t kRingSmemLimit = 232448 - 5120;

// Shape of the ring pipeline for head dim D, group G and window W > 0: tile
// tokens TM, key blocks per window NWIN (BN = NWIN * TM keys), S column
// stride, Q stages NQ and ring blocks NB. False when the window's keys for
// one tile do not fit one MMA (BN <= 192), the S/P double buffer plus O do
// not fit TMEM, or the stages do not fit shared memory.
struct RingShape {
  int TM, KB, NWIN, BN, scol, NQ, NB;
};
bool ring_shape(int D, int G, int window, RingShape* r) {
  if (window <= 0 || !(G == 2 || G == 4 || G == 8)) return false;
  r->TM = 128 / G;
  r->KB = (window - 1 + r->TM - 1) / r->TM;
  r->NWIN = r->KB + 1;
  r->BN = r->NWIN * r->TM;
  r->scol = round_up(r->BN, 32);
  if (r->BN > 16 * swa::kRingMaxBN16 || 2 * r->scol + D > 512) return false;
  r->NQ = 3;
  r->NB = std::min(swa::kRingMaxBlocks, r->NWIN + 3);
  while (swa::ring_smem_bytes(D, r->TM, r->NB, r->NQ) > kRingSmemLimit) {
    if (r->NB > r->NWIN + 1) --r->NB;
    else if (r->NQ > 2) --r->NQ;
    else return false;
  }
  return r->NB > r->NWIN;
}

// Sliding-window prefill on the persistent ring pipeline when ring_shape
// accepts the shape; SWA_ERR_UNSUPPORTED (nothing launched) otherwise. The
// launch has one CTA per work unit, and CTAs that finish early take over the
// units of CTAs not yet started by cancelling their launch (cluster launch
// control): no device memory and no state between calls. With `noalloc` >= 0
// the kernel instead draws its ranges from the counter in static slot
// `noalloc`, on one CTA per SM. With `rope` the kernel rotates q and k itself
// (and writes the ring it names).
template <int D>
int launch_prefill_ring(const void* q, const void* k, const void* v, const int32_t* cu,
                        int num_seqs, int total, int Hq, int Hkv, int window, const float* sink,
                        float scale, void* o, float* lse, cudaStream_t st, int noalloc,
                        const swa::RopeArgs* rope = nullptr) {
  const int G = Hq / Hkv;
  RingShape rs;
  if (!ring_shape(D, G, window, &rs)) return SWA_ERR_UNSUPPORTED;
  const int TM = rs.TM, BN = rs.BN;
  unsigned int* slot = nullptr;
  if (noalloc >= 0 && noalloc_slot(noalloc, &slot) != SWA_OK) return SWA_ERR_CUDA;
  swa::RingParams p;
  p.cu_seqlens = cu;
  p.num_seqs = num_seqs;
  p.total = total;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.TM = TM;
  p.window = window;
  p.KB = rs.KB;
  p.NWIN = rs.NWIN;
  p.NB = rs.NB;
  p.NQ = rs.NQ;
  p.n_tok_tiles = (total + TM - 1) / TM;
  p.n_tiles = p.n_tok_tiles * Hkv;
  p.sink = sink;
  p.scale_log2 = scale * swa::kLog2e;
  p.lse = lse;
  p.q_box_bytes = 128u * TM * G;
  p.s_stride = static_cast<uint32_t>(rs.scol);
  p.o_col = static_cast<uint32_t>(2 * rs.scol);

  CUtensorMap tq, tk, tv, to;
  if (encode_3d(&tq, q, D, Hq, total, 64, G, TM) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tk, k, D, Hkv, total, 64, 1, TM) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tv, v, D, Hkv, total, 64, 1, TM) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&to, o, D, Hq, total, 64, G, TM) != SWA_OK) return SWA_ERR_CUDA;

  const size_t smem = swa::ring_smem_bytes(D, TM, rs.NB, rs.NQ);
  const int nsm = sm_count();
  if (nsm <= 0) return cuda_fail("cudaDeviceGetAttribute(multiprocessor count)", 0);
  p.sched = slot;
  const int units = ring_schedule(p.n_tiles, nsm, slot != nullptr, &p);
  const int grid = slot != nullptr ? p.n_static : units;
  static const swa::RopeArgs no_rope{};
  switch (BN / 16) {
#define SWA_RING_CASE(N)                                                              \
  case N:                                                                             \
    return rope ? run_ring<D, N, true>(tq, tk, tv, to, p, *rope, smem, grid, st)      \
                : run_ring<D, N, false>(tq, tk, tv, to, p, no_rope, smem, grid, st);
    SWA_RING_CASE(1) SWA_RING_CASE(2) SWA_RING_CASE(3) SWA_RING_CASE(4) SWA_RING_CASE(5)
    SWA_RING_CASE(6) SWA_RING_CASE(7) SWA_RING_CASE(8) SWA_RING_CASE(9) SWA_RING_CASE(10)
    SWA_RING_CASE(11) SWA_RING_CASE(12)
#undef SWA_RING_CASE
    default:
      return SWA_ERR_UNSUPPORTED;
  }
}

size_t g_attr_chunked[2][kMaxDevices];

// Global attention, and sliding windows too wide for the ring pipeline, on the
// persistent chunked pipeline (128-key chunks) when the query heads of one kv
// head pack a 128-row tile (G divides 128). SWA_ERR_UNSUPPORTED otherwise.
template <int D>
int launch_prefill_chunked(const void* q, const void* k, const void* v, const int32_t* cu,
                           int num_seqs, int total, int Hq, int Hkv, int window,
                           const float* sink, float scale, void* o, float* lse, cudaStream_t st) {
  const int G = Hq / Hkv;
  if (G < 1 || 128 % G != 0) return SWA_ERR_UNSUPPORTED;
  const int TM = 128 / G;
  swa::ChunkParams p;
  p.cu_seqlens = cu;
  p.num_seqs = num_seqs;
  p.total = total;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.TM = TM;
  p.window = window;
  p.n_tok_tiles = (total + TM - 1) / TM;
  const long long n_tiles = static_cast<long long>(p.n_tok_tiles) * Hkv;
  if (n_tiles > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  p.n_tiles = static_cast<int>(n_tiles);
  p.sink = sink;
  p.scale_log2 = scale * swa::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.q_box_bytes = 128u * TM * G;

  CUtensorMap tq, tk, tv;
  if (encode_3d(&tq, q, D, Hq, total, 64, G, TM) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tk, k, D, Hkv, total, 64, 1, swa::kChunkKeys) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tv, v, D, Hkv, total, 64, 1, swa::kChunkKeys) != SWA_OK) return SWA_ERR_CUDA;

  const size_t smem = swa::chunked_smem_bytes(D);
  auto kern = swa::prefill_chunked_kernel<D>;
  if (ensure_smem_attr(kern, smem, g_attr_chunked[D == 128]) != SWA_OK) return SWA_ERR_CUDA;
  const int nsm = sm_count();
  if (nsm <= 0) return cuda_fail("cudaDeviceGetAttribute(multiprocessor count)", 0);
  const int grid = std::min(nsm, p.n_tiles);
  kern<<<grid, swa::kChunkThreads, smem, st>>>(tq, tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("chunked prefill launch", e);
}

// Dynamic shared memory of the fallback prefill kernel for key chunks of BN.
size_t prefill_smem_bytes(int D, int BN) {
  return 1024 + (D / 64) * 16384 + 2 * (D / 64) * static_cast<size_t>(BN) * 128 +
         static_cast<size_t>((BN + 63) / 64) * 16384;
}

template <int D>
int launch_prefill(const void* q, const void* k, const void* v, const int32_t* cu, int num_seqs,
                   int total, int Hq, int Hkv, int window, const float* sink, float scale,
                   void* o, float* lse, cudaStream_t st) {
  const int G = Hq / Hkv;
  const int TM = 128 / G;
  int BN;
  if (window > 0 && window + TM - 1 <= 256)
    BN = round_up(window + TM - 1, 16);
  else
    BN = 128;
  swa::PrefillParams p;
  p.cu_seqlens = cu;
  p.num_seqs = num_seqs;
  p.total = total;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.TM = TM;
  p.window = window;
  p.BN = BN;
  p.n_tok_tiles = (total + TM - 1) / TM;
  p.reverse = window > 0 ? 0 : 1;
  p.sink = sink;
  p.scale_log2 = scale * swa::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.q_box_bytes = 128u * TM * G;
  p.o_col = static_cast<uint32_t>(round_up(BN, 32));
  p.tmem_cols = static_cast<uint32_t>(next_pow2(static_cast<int>(p.o_col) + D));
  if (p.tmem_cols > 512) return SWA_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  if (encode_3d(&tq, q, D, Hq, total, 64, G, TM) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tk, k, D, Hkv, total, 64, 1, BN) != SWA_OK) return SWA_ERR_CUDA;
  if (encode_3d(&tv, v, D, Hkv, total, 64, 1, BN) != SWA_OK) return SWA_ERR_CUDA;

  const size_t smem = prefill_smem_bytes(D, BN);
  auto kern = swa::prefill_sm100_kernel<D>;
  if (ensure_smem_attr(kern, smem, D == 64 ? g_attr_prefill64 : g_attr_prefill128) != SWA_OK)
    return SWA_ERR_CUDA;
  const long long grid = static_cast<long long>(p.n_tok_tiles) * Hkv;
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  kern<<<static_cast<unsigned>(grid), 128, smem, st>>>(tq, tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("prefill launch", e);
}

template <int D, int MT, int NWP, bool KV8>
int launch_decode(const swa::DecodeFp8Params& p, cudaStream_t st) {
  // boxes of 64 head-dim columns: Q [G heads x n_q tokens], ring [W rows],
  // new rows [n_q rows], of one (sequence, kv head); an FP8 ring as one box
  // of W rows x D codes
  CUtensorMap tq, tkr, tkn, tvr, tvn, to;
  const uint32_t G = static_cast<uint32_t>(p.G), nq = static_cast<uint32_t>(p.n_q);
  const uint32_t W = static_cast<uint32_t>(p.W);
  const bool ring_ok =
      KV8 ? (encode_u8_4d(&tkr, p.k_ring, D, p.Hkv, p.W, p.B, D, 1, W, 1) == SWA_OK &&
             encode_u8_4d(&tvr, p.v_ring, D, p.Hkv, p.W, p.B, D, 1, W, 1) == SWA_OK)
          : (encode_4d(&tkr, p.k_ring, D, p.Hkv, p.W, p.B, 64, 1, W, 1) == SWA_OK &&
             encode_4d(&tvr, p.v_ring, D, p.Hkv, p.W, p.B, 64, 1, W, 1) == SWA_OK);
  if (!ring_ok || encode_4d(&tq, p.q, D, p.Hq, p.n_q, p.B, 64, G, nq, 1) != SWA_OK ||
      encode_4d(&tkn, p.k_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK ||
      encode_4d(&tvn, p.v_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK ||
      encode_4d(&to, p.o, D, p.Hq, p.n_q, p.B, 64, G, nq, 1) != SWA_OK)
    return SWA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hkv;
  auto& attr = g_attr_dec[KV8][D == 128][MT - 1][NWP == swa::kDecodeLargeWarps];
  if constexpr (KV8) {
    const size_t smem = swa::decode_fp8_smem_bytes(D, p.KP, p.W8, NWP);
    auto kern = swa::decode_fp8_sm100_kernel<D, MT, NWP>;
    if (ensure_smem_attr(kern, smem, attr) != SWA_OK) return SWA_ERR_CUDA;
    kern<<<grid, NWP * 32, smem, st>>>(tq, tkr, tkn, tvr, tvn, to, p);
  } else {  // the bf16 ring (the kernel takes the DecodeParams part)
    const size_t smem = swa::decode_smem_bytes(D, p.KP, NWP);
    auto kern = swa::decode_sm100_kernel<D, MT, NWP>;
    if (ensure_smem_attr(kern, smem, attr) != SWA_OK)
      return SWA_ERR_CUDA;
    // the whole unified L1 / shared array as shared memory, so that five
    // 4-warp CTAs fit an SM
    if (ensure_carveout(kern, g_carve_dec[D == 128][MT - 1][NWP == swa::kDecodeLargeWarps]) !=
        SWA_OK)
      return SWA_ERR_CUDA;
    kern<<<grid, NWP * 32, smem, st>>>(tq, tkr, tkn, tvr, tvn, to, p);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("decode launch", e);
}

// Key rows of the tcgen05 decode: the ring, the new rows from W8, padded to
// the MMA's N granule of 16.
int decode_tc_kp(const swa::DecodeParams& p) { return round_up(p.W8 + p.n_q, 16); }

// The tcgen05 decode takes a bf16 ring whose keys fit its softmax registers
// and whose slots fit one CTA's shared memory (227 KB with the barriers).
bool decode_tc_fits(const swa::DecodeParams& p, int D) {
  const int KP = decode_tc_kp(p);
  return KP <= swa::kDecTcMaxKP && swa::decode_tc_smem_bytes(D, KP) + 1024 <= 232448;
}

template <int D>
int launch_decode_tc(const swa::DecodeParams& p, cudaStream_t st) {
  // the same boxes as the one-CTA-per-unit kernel
  CUtensorMap tq, tkr, tkn, tvr, tvn, to;
  const uint32_t G = static_cast<uint32_t>(p.G), nq = static_cast<uint32_t>(p.n_q);
  const uint32_t W = static_cast<uint32_t>(p.W);
  if (encode_4d(&tkr, p.k_ring, D, p.Hkv, p.W, p.B, 64, 1, W, 1) != SWA_OK ||
      encode_4d(&tvr, p.v_ring, D, p.Hkv, p.W, p.B, 64, 1, W, 1) != SWA_OK ||
      encode_4d(&tq, p.q, D, p.Hq, p.n_q, p.B, 64, G, nq, 1) != SWA_OK ||
      encode_4d(&tkn, p.k_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK ||
      encode_4d(&tvn, p.v_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK ||
      encode_4d(&to, p.o, D, p.Hq, p.n_q, p.B, 64, G, nq, 1) != SWA_OK)
    return SWA_ERR_CUDA;
  swa::DecodeTcParams tp;
  tp.d = p;
  tp.d.KP = decode_tc_kp(p);
  tp.s_stride = static_cast<uint32_t>(round_up(tp.d.KP, 32));
  tp.o_col = 2 * tp.s_stride;
  tp.tmem_cols = static_cast<uint32_t>(next_pow2(static_cast<int>(tp.o_col) + D));
  if (tp.tmem_cols > 512) return SWA_ERR_UNSUPPORTED;
  const size_t smem = swa::decode_tc_smem_bytes(D, tp.d.KP);
  auto kern = swa::decode_tc_sm100_kernel<D>;
  if (ensure_smem_attr(kern, smem, g_attr_dec_tc[D == 128]) != SWA_OK) return SWA_ERR_CUDA;
  // one CTA per (sequence, kv head); the CTAs that run take over the units of
  // those that have not started (cluster launch control)
  const unsigned grid = static_cast<unsigned>(p.B) * static_cast<unsigned>(p.Hkv);
  kern<<<grid, swa::kDecTcThreads, smem, st>>>(tq, tkr, tkn, tvr, tvn, to, tp);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("tcgen05 decode launch", e);
}

template <bool KV8>
int pick_decode(const swa::DecodeFp8Params& p, int D, cudaStream_t st) {
  if constexpr (!KV8) {
    if (decode_tc_fits(p, D))
      return D == 64 ? launch_decode_tc<64>(p, st) : launch_decode_tc<128>(p, st);
  }
  const bool two = p.R > 16;
  // 4 warps up to 160 keys, else 8
  if (p.KP <= swa::kDecodeSmallMaxKP) {
    constexpr int S = swa::kDecodeSmallWarps;
    if (D == 64)
      return two ? launch_decode<64, 2, S, KV8>(p, st) : launch_decode<64, 1, S, KV8>(p, st);
    return two ? launch_decode<128, 2, S, KV8>(p, st) : launch_decode<128, 1, S, KV8>(p, st);
  }
  constexpr int L = swa::kDecodeLargeWarps;
  if (D == 64)
    return two ? launch_decode<64, 2, L, KV8>(p, st) : launch_decode<64, 1, L, KV8>(p, st);
  return two ? launch_decode<128, 2, L, KV8>(p, st) : launch_decode<128, 1, L, KV8>(p, st);
}

// swa_sink_attn_decode (kv_scale NULL: bf16 ring) and
// swa_sink_attn_decode_fp8kv (E4M3 ring with per-kv-head scales).
int decode_impl(const void* q, const void* k_new, const void* v_new, const void* k_ring,
                const void* v_ring, const float* kv_scale, const int32_t* pos, int B, int n_q,
                int Hq, int Hkv, int D, int W, const float* sink, float softmax_scale, void* o,
                float* lse, void* stream) {
  if (B < 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || W <= 0) return SWA_ERR_SHAPE;
  if (Hq % Hkv != 0) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (n_q > 8 || W > 256 || n_q * (Hq / Hkv) > 32) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  if (!q || !k_new || !v_new || !k_ring || !v_ring || !pos || !o) return SWA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ring) ||
      !aligned16(v_ring) || !aligned16(o))
    return SWA_ERR_ALIGN;
  if (!aligned4(pos) || (sink && !aligned4(sink)) || (lse && !aligned4(lse)) ||
      (kv_scale && !aligned4(kv_scale)))
    return SWA_ERR_ALIGN;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    softmax_scale = 1.0f / std::sqrt(static_cast<float>(D));
  swa::DecodeFp8Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_ring = static_cast<const __nv_bfloat16*>(k_ring);
  p.v_ring = static_cast<const __nv_bfloat16*>(v_ring);
  p.kv_scale = kv_scale;
  p.pos = pos;
  p.B = B;
  p.n_q = n_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.W = W;
  p.R = n_q * p.G;
  // the new tokens' columns start at a multiple of 8 (16 for an FP8 ring,
  // whose kernel gives them a 16-key block of their own)
  p.W8 = round_up(W, kv_scale ? 16 : 8);
  // keys padded to 16 for the FP8 ring's k16 steps; to 8 for the bf16 ring
  // (its PV ends with a k8 step), which keeps its CTA small enough for five
  // per SM
  p.KP = round_up(p.W8 + n_q, kv_scale ? 16 : 8);
  p.sink = sink;
  p.scale_log2 = softmax_scale * swa::kLog2e;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  if (static_cast<long long>(B) * Hkv > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return kv_scale ? pick_decode<true>(p, D, st) : pick_decode<false>(p, D, st);
}

// Raise the shared-memory limit of every prefill kernel swa_sink_attn_fwd can
// launch (the ring kernel for each window size class, the chunked kernel and
// the fallback kernel, both head dims) to the most it can ask for, on the
// current device.
template <int D, int... N>
int raise_ring_limits(std::integer_sequence<int, N...>) {
  int rc = SWA_OK;
  ((rc = rc != SWA_OK ? rc
                      : ensure_smem_attr(swa::prefill_swa_ring_kernel<D, N + 1, false>,
                                         kRingSmemLimit, g_attr_ring[0][D == 128][N + 1])),
   ...);
  return rc;
}

int raise_prefill_smem_limits() {
  using Classes = std::make_integer_sequence<int, swa::kRingMaxBN16>;
  if (raise_ring_limits<64>(Classes{}) != SWA_OK || raise_ring_limits<128>(Classes{}) != SWA_OK)
    return SWA_ERR_CUDA;
  if (ensure_smem_attr(swa::prefill_chunked_kernel<64>, swa::chunked_smem_bytes(64),
                       g_attr_chunked[0]) != SWA_OK ||
      ensure_smem_attr(swa::prefill_chunked_kernel<128>, swa::chunked_smem_bytes(128),
                       g_attr_chunked[1]) != SWA_OK)
    return SWA_ERR_CUDA;
  if (ensure_smem_attr(swa::prefill_sm100_kernel<64>, prefill_smem_bytes(64, 256),
                       g_attr_prefill64) != SWA_OK ||
      ensure_smem_attr(swa::prefill_sm100_kernel<128>, prefill_smem_bytes(128, 256),
                       g_attr_prefill128) != SWA_OK)
    return SWA_ERR_CUDA;
  return SWA_OK;
}

// swa_sink_attn_fwd and swa_sink_attn_fwd_noalloc: validation and kernel
// choice. noalloc: the static scheduler slot of the ring kernel, or -1 for
// the library's own buffer.
int fwd_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
             int num_seqs, int max_seqlen, int total_tokens, int Hq, int Hkv, int D, int window,
             const float* sink, float softmax_scale, void* o, float* lse, void* stream,
             int noalloc) {
  if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0)
    return SWA_ERR_SHAPE;
  if (Hq % Hkv != 0) return SWA_ERR_SHAPE;
  if (total_tokens > 0 && num_seqs == 0) return SWA_ERR_SHAPE;
  if (max_seqlen > total_tokens) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 128) return SWA_ERR_UNSUPPORTED;
  if (total_tokens == 0) return SWA_OK;
  if (!q || !k || !v || !o || !cu_seqlens) return SWA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SWA_ERR_ALIGN;
  if (!aligned4(cu_seqlens) || (sink && !aligned4(sink)) || (lse && !aligned4(lse)))
    return SWA_ERR_ALIGN;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    softmax_scale = 1.0f / std::sqrt(static_cast<float>(D));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // sliding windows: the persistent ring pipeline when the shape allows it
  if (window > 0) {
    const int rc = D == 64 ? launch_prefill_ring<64>(q, k, v, cu_seqlens, num_seqs,
                                                     total_tokens, Hq, Hkv, window, sink,
                                                     softmax_scale, o, lse, st, noalloc)
                           : launch_prefill_ring<128>(q, k, v, cu_seqlens, num_seqs,
                                                      total_tokens, Hq, Hkv, window, sink,
                                                      softmax_scale, o, lse, st, noalloc);
    if (rc != SWA_ERR_UNSUPPORTED) return rc;
  }
  {
    const int rc = D == 64 ? launch_prefill_chunked<64>(q, k, v, cu_seqlens, num_seqs,
                                                        total_tokens, Hq, Hkv, window, sink,
                                                        softmax_scale, o, lse, st)
                           : launch_prefill_chunked<128>(q, k, v, cu_seqlens, num_seqs,
                                                         total_tokens, Hq, Hkv, window, sink,
                                                         softmax_scale, o, lse, st);
    if (rc != SWA_ERR_UNSUPPORTED) return rc;
  }
  if (D == 64)
    return launch_prefill<64>(q, k, v, cu_seqlens, num_seqs, total_tokens, Hq, Hkv, window, sink,
                              softmax_scale, o, lse, st);
  return launch_prefill<128>(q, k, v, cu_seqlens, num_seqs, total_tokens, Hq, Hkv, window, sink,
                             softmax_scale, o, lse, st);
}

// ---- prefill with the rotary embedding ------------------------------------------
// Two routes. With a workspace: a standalone pass writes rotated copies of q
// and k there (q then k, the k copy 256-byte aligned), then the plain prefill
// runs on them; the prefill kernels read q and k through TMA straight into
// the MMAs. Without one (ring shapes only): the ring kernel rotates each Q
// tile and K block in shared memory. The first is the faster for the 32K SWA
// layer (the rotation inside the ring kernel lengthens its epilogue's
// critical path more than a separate pass over q and k costs); the second
// needs no memory beyond the call's inputs and outputs.
size_t rope_k_offset(int total, int Hq, int D) {
  const size_t qb = static_cast<size_t>(total) * Hq * D * 2;
  return (qb + 255) / 256 * 256;
}

// The workspace of the two-pass route (rotated q, then k). Every shape can
// take that route; shapes the ring kernel takes can also rotate in shared
// memory without a workspace (a call given none).
size_t rope_workspace_bytes(int total, int Hq, int Hkv, int D, int window) {
  (void)window;
  if (total <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (D != 64 && D != 128)) return 0;
  return rope_k_offset(total, Hq, D) + static_cast<size_t>(total) * Hkv * D * 2;
}

int fwd_rope_impl(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                  int num_seqs, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                  int window, const float* sink, float softmax_scale, float rope_base,
                  int rope_interleaved, const int32_t* pos0, void* k_ring, void* v_ring,
                  int ring_W, void* workspace, size_t workspace_bytes, void* o, float* lse,
                  void* stream) {
  if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0)
    return SWA_ERR_SHAPE;
  if (Hq % Hkv != 0) return SWA_ERR_SHAPE;
  if (total_tokens > 0 && num_seqs == 0) return SWA_ERR_SHAPE;
  if (max_seqlen > total_tokens) return SWA_ERR_SHAPE;
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return SWA_ERR_SHAPE;
  if (rope_interleaved != 0 && rope_interleaved != 1) return SWA_ERR_SHAPE;
  if ((k_ring == nullptr) != (v_ring == nullptr)) return SWA_ERR_NULL;
  if (k_ring != nullptr && ring_W < 1) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (Hq / Hkv > 128) return SWA_ERR_UNSUPPORTED;
  if (total_tokens == 0) return SWA_OK;
  if (!q || !k || !v || !o || !cu_seqlens) return SWA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SWA_ERR_ALIGN;
  if (k_ring != nullptr && (!aligned16(k_ring) || !aligned16(v_ring))) return SWA_ERR_ALIGN;
  if (!aligned4(cu_seqlens) || (sink && !aligned4(sink)) || (lse && !aligned4(lse)) ||
      (pos0 && !aligned4(pos0)))
    return SWA_ERR_ALIGN;
  // route: rotate into the workspace and run the plain prefill (when the
  // caller gives one), else rotate in the ring kernel's shared memory (ring
  // shapes only)
  const size_t need = rope_workspace_bytes(total_tokens, Hq, Hkv, D, window);
  RingShape rs_probe;
  const bool fused = workspace == nullptr && ring_shape(D, Hq / Hkv, window, &rs_probe);
  if (!fused) {
    if (workspace == nullptr) return SWA_ERR_NULL;
    if (workspace_bytes < need) return SWA_ERR_SHAPE;
    if (!aligned16(workspace)) return SWA_ERR_ALIGN;
  }
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    softmax_scale = 1.0f / std::sqrt(static_cast<float>(D));
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  swa::RopeArgs ra{};
  ra.pos0 = pos0;
  ra.interleaved = rope_interleaved;
  // theta_c / (2 pi) = base^(-2c/D) / (2 pi), split into two floats
  for (int c = 0; c < D / 2; ++c) {
    const double f = std::pow(static_cast<double>(rope_base), -2.0 * c / D) /
                     (2.0 * 3.14159265358979323846);
    ra.f_hi[c] = static_cast<float>(f);
    ra.f_lo[c] = static_cast<float>(f - static_cast<double>(ra.f_hi[c]));
  }
  ra.k_ring = static_cast<__nv_bfloat16*>(k_ring);
  ra.v_ring = static_cast<__nv_bfloat16*>(v_ring);
  ra.ring_W = k_ring != nullptr ? ring_W : 0;

  if (fused) {  // the ring kernel, rotating in shared memory
    return D == 64 ? launch_prefill_ring<64>(q, k, v, cu_seqlens, num_seqs, total_tokens, Hq,
                                             Hkv, window, sink, softmax_scale, o, lse, st, -1,
                                             &ra)
                   : launch_prefill_ring<128>(q, k, v, cu_seqlens, num_seqs, total_tokens, Hq,
                                              Hkv, window, sink, softmax_scale, o, lse, st, -1,
                                              &ra);
  }
  // rotate into the workspace, then the plain prefill on the rotated copies
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  swa::RopePassParams pp;
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.q_out = reinterpret_cast<__nv_bfloat16*>(ws);
  pp.k_out = reinterpret_cast<__nv_bfloat16*>(ws + rope_k_offset(total_tokens, Hq, D));
  pp.cu_seqlens = cu_seqlens;
  pp.num_seqs = num_seqs;
  pp.total = total_tokens;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  if (D == 64) swa::rope_pass_kernel<64><<<total_tokens, 128, 0, st>>>(pp, ra);
  else swa::rope_pass_kernel<128><<<total_tokens, 128, 0, st>>>(pp, ra);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("rope pass launch", e);
  const void* qr = pp.q_out;
  const void* kr = pp.k_out;
  if (window > 0) {
    const int rc = D == 64 ? launch_prefill_ring<64>(qr, kr, v, cu_seqlens, num_seqs,
                                                     total_tokens, Hq, Hkv, window, sink,
                                                     softmax_scale, o, lse, st, -1)
                           : launch_prefill_ring<128>(qr, kr, v, cu_seqlens, num_seqs,
                                                      total_tokens, Hq, Hkv, window, sink,
                                                      softmax_scale, o, lse, st, -1);
    if (rc != SWA_ERR_UNSUPPORTED) return rc;
  }
  {
    const int rc = D == 64 ? launch_prefill_chunked<64>(qr, kr, v, cu_seqlens, num_seqs,
                                                        total_tokens, Hq, Hkv, window, sink,
                                                        softmax_scale, o, lse, st)
                           : launch_prefill_chunked<128>(qr, kr, v, cu_seqlens, num_seqs,
                                                         total_tokens, Hq, Hkv, window, sink,
                                                         softmax_scale, o, lse, st);
    if (rc != SWA_ERR_UNSUPPORTED) return rc;
  }
  if (D == 64)
    return launch_prefill<64>(qr, kr, v, cu_seqlens, num_seqs, total_tokens, Hq, Hkv, window,
                              sink, softmax_scale, o, lse, st);
  return launch_prefill<128>(qr, kr, v, cu_seqlens, num_seqs, total_tokens, Hq, Hkv, window, sink,
                             softmax_scale, o, lse, st);
}

// ---- backward ---------------------------------------------------------------------
size_t bwd_workspace_bytes(int total, int Hq) {
  if (total <= 0 || Hq <= 0) return 0;
  return (static_cast<size_t>(total) * Hq * sizeof(float) + 255) / 256 * 256;
}

size_t g_attr_bt_dq[2][kMaxDevices], g_attr_bt_dkdv[2][kMaxDevices];

// Backward on tcgen05: the dq pipeline (which also writes Delta and adds up
// dsink), then the dk/dv pipeline (persistent, one CTA per SM).
template <int D>
int launch_bwd(const swa::BwdParams& b, cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  const int nsm = sm_count();
  if (nsm <= 0) return SWA_ERR_CUDA;
  swa::BtParams p;
  p.cu_seqlens = b.cu_seqlens;
  p.num_seqs = b.num_seqs;
  p.total = b.total;
  p.Hq = b.Hq;
  p.Hkv = b.Hkv;
  p.G = b.G;
  p.lg = 0;
  while ((1 << p.lg) < b.G) ++p.lg;  // G divides 64: a power of two
  p.window = b.window;
  p.TM = swa::kBtQRows / b.G;
  p.TOK = swa::kBtRows / b.G;
  p.lse = b.lse;
  p.delta = b.delta;
  p.o = b.o;
  p.dout = b.dout;
  p.sink = b.sink;
  p.dsink = b.dsink;
  p.scale = b.scale;
  p.scale_log2 = b.scale_log2;
  p.dq = b.dq;
  p.dk = b.dk;
  p.dv = b.dv;
  p.q_box_bytes = 64u * 2u * swa::kBtQRows;
  const uint32_t G = static_cast<uint32_t>(b.G);
  {
    CUtensorMap tq, tdo, tk, tv;
    if (encode_3d(&tq, b.q, D, b.Hq, b.total, 64, G, p.TM) != SWA_OK ||
        encode_3d(&tdo, b.dout, D, b.Hq, b.total, 64, G, p.TM) != SWA_OK ||
        encode_3d(&tk, b.k, D, b.Hkv, b.total, 64, 1, swa::kBtChunk) != SWA_OK ||
        encode_3d(&tv, b.v, D, b.Hkv, b.total, 64, 1, swa::kBtChunk) != SWA_OK)
      return SWA_ERR_CUDA;
    p.n_units = (b.total + p.TM - 1) / p.TM;
    const long long tiles = static_cast<long long>(p.n_units) * b.Hkv;
    if (tiles > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
    p.n_tiles = static_cast<int>(tiles);
    auto kern = swa::bwd_dq_tc_kernel<D>;
    const size_t smem = swa::bt_dq_smem_bytes<D>();
    if (ensure_smem_attr(kern, smem, g_attr_bt_dq[D == 128]) != SWA_OK) return SWA_ERR_CUDA;
    kern<<<std::min(p.n_tiles, nsm), swa::kBtThreads, smem, st>>>(tq, tdo, tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("backward dq launch", e);
  }
  {
    CUtensorMap tk, tv, tq, tdo;
    if (encode_3d(&tk, b.k, D, b.Hkv, b.total, 64, 1, swa::kBtKeys) != SWA_OK ||
        encode_3d(&tv, b.v, D, b.Hkv, b.total, 64, 1, swa::kBtKeys) != SWA_OK ||
        encode_3d(&tq, b.q, D, b.Hq, b.total, 64, G, p.TOK) != SWA_OK ||
        encode_3d(&tdo, b.dout, D, b.Hq, b.total, 64, G, p.TOK) != SWA_OK)
      return SWA_ERR_CUDA;
    p.n_units = (b.total + swa::kBtKeys - 1) / swa::kBtKeys;
    const long long tiles = static_cast<long long>(p.n_units) * b.Hkv;
    if (tiles > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
    p.n_tiles = static_cast<int>(tiles);
    auto kern = swa::bwd_dkdv_tc_kernel<D>;
    const size_t smem = swa::bt_dkdv_smem_bytes<D>();
    if (ensure_smem_attr(kern, smem, g_attr_bt_dkdv[D == 128]) != SWA_OK) return SWA_ERR_CUDA;
    kern<<<std::min(p.n_tiles, nsm), swa::kBtThreads, smem, st>>>(tk, tv, tq, tdo, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("backward dk/dv launch", e);
  }
  return SWA_OK;
}

int bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
             int total_tokens, int Hq, int Hkv, int D, int window, const float* sink,
             float softmax_scale, void* dq, void* dk, void* dv, float* dsink, void* workspace,
             size_t workspace_bytes, void* stream) {
  if (num_seqs < 0 || max_seqlen < 0 || total_tokens < 0 || Hq <= 0 || Hkv <= 0)
    return SWA_ERR_SHAPE;
  if (Hq % Hkv != 0) return SWA_ERR_SHAPE;
  if (total_tokens > 0 && num_seqs == 0) return SWA_ERR_SHAPE;
  if (max_seqlen > total_tokens) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (swa::kBtRows % (Hq / Hkv) != 0) return SWA_ERR_UNSUPPORTED;  // G divides 64
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total_tokens == 0) {
    if (dsink != nullptr) {
      if (!aligned4(dsink)) return SWA_ERR_ALIGN;
      const cudaError_t e = cudaMemsetAsync(dsink, 0, sizeof(float) * Hq, st);
      if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(dsink)", e);
    }
    return SWA_OK;
  }
  if (!q || !k || !v || !o || !dout || !lse || !cu_seqlens || !dq || !dk || !dv)
    return SWA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SWA_ERR_ALIGN;
  if (!aligned4(cu_seqlens) || !aligned4(lse) || (sink && !aligned4(sink)) ||
      (dsink && !aligned4(dsink)))
    return SWA_ERR_ALIGN;
  if (workspace == nullptr) return SWA_ERR_NULL;
  if (workspace_bytes < bwd_workspace_bytes(total_tokens, Hq)) return SWA_ERR_SHAPE;
  if (!aligned16(workspace)) return SWA_ERR_ALIGN;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    softmax_scale = 1.0f / std::sqrt(static_cast<float>(D));
  if (dsink != nullptr) {  // the dq kernel adds into it
    const cudaError_t e = cudaMemsetAsync(dsink, 0, sizeof(float) * Hq, st);
    if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(dsink)", e);
  }
  swa::BwdParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.lse = lse;
  p.cu_seqlens = cu_seqlens;
  p.num_seqs = num_seqs;
  p.total = total_tokens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.window = window;
  p.sink = sink;
  p.scale = softmax_scale;
  p.scale_log2 = softmax_scale * swa::kLog2e;
  p.delta = static_cast<float*>(workspace);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dsink = dsink;
  return D == 64 ? launch_bwd<64>(p, st) : launch_bwd<128>(p, st);
}

// ---- split-KV decode ------------------------------------------------------------
// Ranges per (sequence, kv head) and their length: enough CTAs for a few waves
// (a fixed target, so that the workspace size does not depend on the device),
// no more ranges than 64-key tiles.
constexpr long long kSplitTargetCtas = 1184;
void split_shape(int B, int Hkv, int W, int max_ctx, int* S, int* chunk) {
  const long long span = std::max(1, std::min(W, max_ctx));
  const long long units = std::max(1LL, static_cast<long long>(B) * Hkv);
  long long s = (kSplitTargetCtas + units - 1) / units;
  s = std::max(1LL, std::min(s, (span + swa::kSplitTile - 1) / swa::kSplitTile));
  long long c = (span + s - 1) / s;
  c = (c + swa::kSplitTile - 1) / swa::kSplitTile * swa::kSplitTile;
  *chunk = static_cast<int>(c);
  *S = static_cast<int>((span + c - 1) / c);
}

size_t split_workspace_bytes(int B, int Hkv, int D, int W, int max_ctx) {
  int S = 0, chunk = 0;
  split_shape(B, Hkv, W, max_ctx, &S, &chunk);
  return static_cast<size_t>(B) * Hkv * S * 32 * (D + 4) * sizeof(float);
}

size_t g_attr_split_tc[2][kMaxDevices];

// The split-KV decode on the tcgen05 kernel: one CTA per (sequence, range, kv
// head), those that run taking over the others' units; then the merge.
template <int D>
int launch_split_tc(const swa::SplitParams& p, const void* q, const void* k_new,
                    const void* v_new, const void* k_cache, const void* v_cache, cudaStream_t st) {
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  const uint32_t G = static_cast<uint32_t>(p.G), nq = static_cast<uint32_t>(p.n_q);
  if (encode_4d(&tq, q, D, p.Hq, p.n_q, p.B, 64, G, nq, 1) != SWA_OK ||
      encode_4d(&tkc, k_cache, D, p.Hkv, p.W, p.B, 64, 1, swa::kSplitTile, 1) != SWA_OK ||
      encode_4d(&tvc, v_cache, D, p.Hkv, p.W, p.B, 64, 1, swa::kSplitTile, 1) != SWA_OK ||
      encode_4d(&tkn, k_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK ||
      encode_4d(&tvn, v_new, D, p.Hkv, p.n_q, p.B, 64, 1, nq, 1) != SWA_OK)
    return SWA_ERR_CUDA;
  // at least half an SM's shared memory, so that one CTA (and its 512 TMEM
  // columns) has the SM
  const size_t smem = std::max<size_t>(swa::split_tc_smem_bytes(D), 120 * 1024);
  auto kern = swa::decode_split_tc_kernel<D>;
  if (ensure_smem_attr(kern, smem, g_attr_split_tc[D == 128]) != SWA_OK) return SWA_ERR_CUDA;
  const long long units = static_cast<long long>(p.B) * p.Hkv;
  if (units * p.S > 0x7fffffffLL || units * p.R > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  kern<<<static_cast<unsigned>(units * p.S), swa::kSplTcThreads, smem, st>>>(tq, tkc, tvc, tkn,
                                                                               tvn, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail("tcgen05 split-KV decode launch", e);
  swa::decode_split_combine_kernel<D><<<static_cast<unsigned>(units * p.R), 32, 0, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? SWA_OK : cuda_fail("split-KV combine launch", e);
}


}  // namespace

extern "C" {

int swa_sink_version(void) { return 100; }

const char* swa_sink_status_string(int status) {
  switch (status) {
    case SWA_OK: return "ok";
    case SWA_ERR_NULL: return "a required pointer is NULL";
    case SWA_ERR_SHAPE: return "a size is negative or inconsistent";
    case SWA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SWA_ERR_ALIGN: return "a pointer is misaligned";
    case SWA_ERR_CUDA: return "a CUDA call failed";
    default: return "unknown status";
  }
}

int swa_sink_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                      int num_seqs, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                      int window, const float* sink, float softmax_scale, void* o, float* lse,
                      void* stream) {
  return fwd_impl(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D, window,
                  sink, softmax_scale, o, lse, stream, -1);
}

int swa_sink_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
                              int total_tokens, int Hq, int Hkv, int D, int window,
                              const float* sink, float softmax_scale, void* o, float* lse,
                              int slot, void* stream) {
  if (slot < 0 || slot >= kNoAllocSlots) return SWA_ERR_SHAPE;
  return fwd_impl(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D, window,
                  sink, softmax_scale, o, lse, stream, slot);
}

size_t swa_sink_attn_bwd_workspace(int total_tokens, int Hq) {
  return bwd_workspace_bytes(total_tokens, Hq);
}

int swa_sink_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, const int32_t* cu_seqlens, int num_seqs,
                      int max_seqlen, int total_tokens, int Hq, int Hkv, int D, int window,
                      const float* sink, float softmax_scale, void* dq, void* dk, void* dv,
                      float* dsink, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, dout, lse, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv,
                  D, window, sink, softmax_scale, dq, dk, dv, dsink, workspace, workspace_bytes,
                  stream);
}

size_t swa_sink_attn_fwd_rope_workspace(int total_tokens, int Hq, int Hkv, int D, int window) {
  return rope_workspace_bytes(total_tokens, Hq, Hkv, D, window);
}

int swa_sink_attn_fwd_rope(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                           int num_seqs, int max_seqlen, int total_tokens, int Hq, int Hkv, int D,
                           int window, const float* sink, float softmax_scale, float rope_base,
                           int rope_interleaved, const int32_t* pos0, void* k_ring, void* v_ring,
                           int ring_W, void* workspace, size_t workspace_bytes, void* o,
                           float* lse, void* stream) {
  return fwd_rope_impl(q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D,
                       window, sink, softmax_scale, rope_base, rope_interleaved, pos0, k_ring,
                       v_ring, ring_W, workspace, workspace_bytes, o, lse, stream);
}

int swa_sink_attn_decode(const void* q, const void* k_new, const void* v_new, const void* k_ring,
                         const void* v_ring, const int32_t* pos, int B, int n_q, int Hq, int Hkv,
                         int D, int W, const float* sink, float softmax_scale, void* o,
                         float* lse, void* stream) {
  return decode_impl(q, k_new, v_new, k_ring, v_ring, nullptr, pos, B, n_q, Hq, Hkv, D, W, sink,
                     softmax_scale, o, lse, stream);
}

int swa_sink_attn_decode_fp8kv(const void* q, const void* k_new, const void* v_new,
                               const void* k_ring, const void* v_ring, const float* kv_scale,
                               const int32_t* pos, int B, int n_q, int Hq, int Hkv, int D, int W,
                               const float* sink, float softmax_scale, void* o, float* lse,
                               void* stream) {
  if (B > 0 && !kv_scale) return SWA_ERR_NULL;
  return decode_impl(q, k_new, v_new, k_ring, v_ring, kv_scale, pos, B, n_q, Hq, Hkv, D, W,
                     sink, softmax_scale, o, lse, stream);
}

size_t swa_sink_decode_splitkv_workspace(int B, int n_q, int Hq, int Hkv, int D, int W,
                                          int max_ctx) {
  if (B < 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || W <= 0 || max_ctx < 0) return 0;
  if (D != 64 && D != 128) return 0;
  return split_workspace_bytes(B, Hkv, D, W, max_ctx);
}

int swa_sink_attn_decode_splitkv(const void* q, const void* k_new, const void* v_new,
                                 const void* k_cache, const void* v_cache, const int32_t* pos,
                                 int B, int n_q, int Hq, int Hkv, int D, int W, int max_ctx,
                                 const float* sink, float softmax_scale, void* o, float* lse,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || W <= 0 || max_ctx < 0) return SWA_ERR_SHAPE;
  if (Hq % Hkv != 0) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (n_q > 8 || n_q * (Hq / Hkv) > 32) return SWA_ERR_UNSUPPORTED;
  if (W % swa::kSplitTile != 0) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o || !workspace)
    return SWA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(o) || !aligned16(workspace))
    return SWA_ERR_ALIGN;
  if (!aligned4(pos) || (sink && !aligned4(sink)) || (lse && !aligned4(lse))) return SWA_ERR_ALIGN;
  if (workspace_bytes < split_workspace_bytes(B, Hkv, D, W, max_ctx)) return SWA_ERR_SHAPE;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    softmax_scale = 1.0f / std::sqrt(static_cast<float>(D));
  swa::SplitParams p;
  p.pos = pos;
  p.B = B;
  p.n_q = n_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.W = W;
  p.R = n_q * p.G;
  split_shape(B, Hkv, W, max_ctx, &p.S, &p.chunk);
  p.sink = sink;
  p.scale_log2 = softmax_scale * swa::kLog2e;
  p.part = static_cast<float*>(workspace);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64) return launch_split_tc<64>(p, q, k_new, v_new, k_cache, v_cache, st);
  return launch_split_tc<128>(p, q, k_new, v_new, k_cache, v_cache, st);
}

int swa_sink_kv_commit(void* k_ring, void* v_ring, const void* k_new, const void* v_new,
                       const int32_t* pos, const int32_t* n_accept, int B, int n_q, int Hkv,
                       int D, int W, void* stream) {
  if (B < 0 || n_q <= 0 || Hkv <= 0 || W <= 0) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  if (!k_ring || !v_ring || !k_new || !v_new || !pos || !n_accept) return SWA_ERR_NULL;
  if (!aligned16(k_ring) || !aligned16(v_ring) || !aligned16(k_new) || !aligned16(v_new))
    return SWA_ERR_ALIGN;
  if (!aligned4(pos) || !aligned4(n_accept)) return SWA_ERR_ALIGN;
  const long long grid = static_cast<long long>(B) * n_q;
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  swa::kv_commit_kernel<<<static_cast<unsigned>(grid), 128, 0, st>>>(
      static_cast<__nv_bfloat16*>(k_ring), static_cast<__nv_bfloat16*>(v_ring),
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), pos,
      n_accept, n_q, Hkv, D, W);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_sink_kv_commit_fp8(void* k_ring, void* v_ring, const void* k_new, const void* v_new,
                           const float* kv_scale, const int32_t* pos, const int32_t* n_accept,
                           int B, int n_q, int Hkv, int D, int W, void* stream) {
  if (B < 0 || n_q <= 0 || Hkv <= 0 || W <= 0) return SWA_ERR_SHAPE;
  if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  if (!k_ring || !v_ring || !k_new || !v_new || !kv_scale || !pos || !n_accept)
    return SWA_ERR_NULL;
  if (!aligned16(k_ring) || !aligned16(v_ring) || !aligned16(k_new) || !aligned16(v_new))
    return SWA_ERR_ALIGN;
  if (!aligned4(kv_scale) || !aligned4(pos) || !aligned4(n_accept)) return SWA_ERR_ALIGN;
  const long long grid = static_cast<long long>(B) * n_q;
  if (grid > 0x7fffffffLL) return SWA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  swa::kv_commit_fp8_kernel<<<static_cast<unsigned>(grid), 128, 0, st>>>(
      static_cast<uint8_t*>(k_ring), static_cast<uint8_t*>(v_ring),
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      kv_scale, pos, n_accept, n_q, Hkv, D, W);
  return cudaGetLastError() == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

int swa_sink_device_error(unsigned int* flags, int clear) {
  if (!flags) return SWA_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return SWA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, swa::g_device_error, sizeof v) != cudaSuccess) return SWA_ERR_CUDA;
  *flags = v;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(swa::g_device_error, &zero, sizeof zero) != cudaSuccess)
      return SWA_ERR_CUDA;
  }
  return SWA_OK;
}

}  // extern "C"
