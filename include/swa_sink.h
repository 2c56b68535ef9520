/*
 * swa_sink.h -- C ABI of libswasink.so: causal GQA attention over a sliding
 * window (or the full prefix) with a per-head learnable attention-sink logit,
 * for NVIDIA B200 (sm_100a).
 *
 * The operation (one query row i of query head h; kv head g = h / (Hq/Hkv)):
 *
 *   a_j  = scale * (q_i . k_j)            over the visible keys j
 *   m    = max(s_h, max_j a_j)
 *   den  = exp(s_h - m) + sum_j exp(a_j - m)
 *   o_i  = sum_j exp(a_j - m) / den * v_j  (the sink carries no value)
 *   lse  = m + ln(den)                     (natural log, sink included)
 *
 * Source: "MiMo-V2-Flash Technical Report" summary (mlpod.com), section 2.2.2
 * "Learnable Attention Sink Bias" (a learnable term in the softmax denominator
 * that lets a row attend to a virtual sink; a max term for stability; the
 * page's equations are stripped, the above is the plain reading of its prose),
 * and section 2.2.1 / TL;DR (window of 128 tokens; SWA and global layers
 * interleaved 5:1). The MiMo-V2 blog review (kokolerk.github.io), section 2.2,
 * states the same sink term. Visible keys for query i: i-W+1 <= j <= i within
 * its own sequence (W keys including itself; the pages do not say whether the
 * query counts, this is the reading taken); W <= 0 means the full causal prefix
 * (the global-attention layers).
 *
 * Conventions for every call
 * --------------------------
 * - All array pointers are DEVICE pointers owned by the caller. bf16 arrays
 *   must be 16-byte aligned (TMA and 16-byte vector loads); int32/fp32 arrays
 *   4-byte. The library allocates no device memory and keeps no device state
 *   between calls, apart from the error flags of swa_sink_device_error() and
 *   the static slots of swa_sink_attn_fwd_noalloc. (The sliding-window
 *   prefill and the bf16-ring decode balance their work with the hardware's
 *   cluster launch control: a CTA that finishes early cancels the launch of
 *   a CTA of the same grid that has not started and does its work. Calls on
 *   any number of streams may run at the same time.) Workspaces, where a
 *   call needs one, are the caller's.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call is asynchronous on that stream; the caller synchronises.
 * - Argument errors are returned as a negative status BEFORE anything is
 *   launched; nothing is written then. A failed launch returns SWA_ERR_CUDA.
 * - The kernels never trap or assert. Each device-side wait has a time limit
 *   (about 2 s); if one expires, or a device-resident argument is out of range
 *   (a negative pos, an n_accept outside [0, n_q]), the kernel records a flag
 *   readable with swa_sink_device_error() and returns.
 * - Thread-safe: the host state (the driver entry point, per-device kernel
 *   attributes) is filled under locks. The first call of a kernel on a
 *   device raises that kernel's shared-memory limit (cudaFuncSetAttribute).
 */
#ifndef SWA_SINK_H
#define SWA_SINK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SWA_API __attribute__((visibility("default")))
#else
#define SWA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SWA_OK = 0,
    SWA_ERR_NULL = -1,        /* a required pointer is NULL                  */
    SWA_ERR_SHAPE = -2,       /* a size is negative or inconsistent          */
    SWA_ERR_UNSUPPORTED = -3, /* valid but not supported (e.g. head_dim 96)  */
    SWA_ERR_ALIGN = -4,       /* a pointer is not aligned as required        */
    SWA_ERR_CUDA = -5         /* a CUDA runtime/driver call failed           */
} swa_status_t;

/*
 * Packed varlen prefill (self-attention, queries and keys share cu_seqlens).
 *
 * Source: section 2.2 of the report summary above (Hybrid SWA: sliding-window
 * layers with W = 128 and global layers), section 2.2.2 (the sink).
 *
 *   q           bf16 [total_tokens, Hq, D], row-major (token, head, dim)
 *   k, v        bf16 [total_tokens, Hkv, D]
 *   cu_seqlens  int32 [num_seqs + 1], device; cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[num_seqs] = total_tokens.
 *               Zero-length sequences are allowed. The host does not read it.
 *   max_seqlen  an upper bound on any sequence length (>= 0); used only to
 *               check sizes.
 *   Hq, Hkv     query / kv heads; Hkv divides Hq; Hq/Hkv <= 128.
 *               Query head h reads kv head h / (Hq/Hkv).
 *   D           head dim: 64 or 128.
 *   window      > 0: key j visible to query i iff i-window+1 <= j <= i;
 *               <= 0: full causal prefix.
 *   sink        fp32 [Hq] device, or NULL for no sink (s_h = -inf).
 *   softmax_scale  <= 0 selects 1/sqrt(D). The sink is not scaled.
 *   o           bf16 [total_tokens, Hq, D] output (round to nearest even).
 *   lse         fp32 [Hq, total_tokens] output in natural-log units, or NULL.
 *
 * Returns SWA_OK or a negative swa_status_t.
 */
SWA_API int swa_sink_attn_fwd(const void *q, const void *k, const void *v,
                      const int32_t *cu_seqlens, int num_seqs, int max_seqlen,
                      int total_tokens, int Hq, int Hkv, int D, int window,
                      const float *sink, float softmax_scale, void *o,
                      float *lse, void *stream);

/*
 * swa_sink_attn_fwd with a software tile scheduler in a static device array.
 *
 * The pages have no counterpart: this is an interface variant. The arguments
 * and the results (bit for bit) are those of swa_sink_attn_fwd, and like it
 * this call allocates no device memory. It is meant for callers that cannot
 * allocate, such as serving runtimes that hand all device memory to their
 * own pool at start-up. The difference lies in the sliding-window
 * kernel's load balancing: here the kernel runs on one CTA per SM and draws
 * its tile ranges from two counters in a static device array of the library
 * (8 slots of two 32-bit words, 64 bytes in all, held by every GPU that loads
 * the library until the process exits) instead of cancelling launches of its
 * own grid.
 *
 *   slot   the static scheduler slot, 0 <= slot < 8. Any other value returns
 *          SWA_ERR_SHAPE before anything is launched (the array holds 8).
 *
 * - Must start at zero: both words of the slot. They are zero when the
 *   library's device code is loaded, and every launch leaves its slot zero
 *   (the launch's last CTA clears it, also after a wait has timed out).
 * - Calls whose kernels overlap in time (other streams, concurrently running
 *   graphs) race on a shared slot and give wrong results: give each of them
 *   its own slot.
 * - The first call on each device does all of this entry point's set-up: it
 *   looks up the array's device address (cudaGetSymbolAddress), raises the
 *   shared-memory limits of every prefill kernel it can launch (all head
 *   dims and windows) and fetches the driver's tensor-map entry point. Later
 *   calls make no set-up call.
 * - Only the sliding-window ring kernel has a scheduler; for shapes it does
 *   not take, the call runs the same kernel as swa_sink_attn_fwd and `slot`
 *   is not used.
 */
SWA_API int swa_sink_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                              const int32_t *cu_seqlens, int num_seqs, int max_seqlen,
                              int total_tokens, int Hq, int Hkv, int D, int window,
                              const float *sink, float softmax_scale, void *o,
                              float *lse, int slot, void *stream);

/*
 * Packed varlen prefill with the rotary position embedding (RoPE) applied to q
 * and k inside the call, and the decode ring of each sequence written from it.
 *
 * Source: the RoPE base per layer type is given in section 3.1 "Data
 * Scheduler" of the report summary above (SWA 10,000; global 640,000, raised
 * to 5,000,000 for the 256K extension); the Q&A of the ICML 2026 talk
 * write-up (hzrcw.cc) says the position index keeps increasing while the
 * window slides. No page prints the rotation: it is the standard rotary
 * embedding over the whole head dim. Pair c (0 <= c < D/2) of a row at
 * absolute position p turns by p * base^(-2c/D):
 *   (x_a, x_b) -> (x_a cos - x_b sin, x_b cos + x_a sin)
 * with (a, b) = (c, c + D/2) when rope_interleaved = 0 ("rotate half"), or
 * (2c, 2c + 1) when rope_interleaved = 1. The rotated q and k are rounded to
 * bf16 (round to nearest even) and then attended exactly as
 * swa_sink_attn_fwd does, so the result is that of rotating, storing in bf16
 * and calling swa_sink_attn_fwd (up to rare 1-ulp differences of a rotated
 * element lying within ~1e-7 relative of a bf16 rounding boundary).
 *
 *   q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D,
 *   window, sink, softmax_scale, o, lse   as for swa_sink_attn_fwd; q and k
 *               are NOT rotated (they are read only).
 *   rope_base   the base (> 0, finite), e.g. 1e4 for SWA layers.
 *   rope_interleaved  0 or 1 (the pairing above).
 *   pos0        int32 [num_seqs] device: the position of each sequence's
 *               first token (token i of sequence s is at pos0[s] + i), or NULL
 *               for 0. Positions must lie in [0, 2^24); others are clamped
 *               and flagged (bit 1 of swa_sink_device_error). The attention
 *               itself still sees only the tokens of this call.
 *   k_ring, v_ring  bf16 [num_seqs, ring_W, Hkv, D], 16-byte aligned, or
 *               both NULL. For the last min(L_s, ring_W) tokens of sequence
 *               s, the rotated key row and the value row of position p go to
 *               slot p mod ring_W (the layout swa_sink_attn_decode reads);
 *               the other slots are not touched. ring_W >= pos0[s] + L_s gives
 *               a plain position-indexed cache (the global layers' layout for
 *               swa_sink_attn_decode_splitkv).
 *   workspace   device memory of swa_sink_attn_fwd_rope_workspace() bytes
 *               (the size of q plus k), 16-byte aligned, owned by the caller.
 *               With it, a separate pass writes rotated copies of q and k
 *               there, then the prefill runs on them: the faster route. NULL
 *               (workspace_bytes ignored) is allowed for sliding windows on
 *               the ring kernel (Hq/Hkv in {2, 4, 8}, window + 128/(Hq/Hkv) - 1
 *               <= 192 keys): that kernel then rotates each Q tile and K block
 *               in shared memory, needing no memory beyond the call's inputs
 *               and outputs. Other shapes (global layers among them) need the
 *               workspace. Calls that overlap in time need separate
 *               workspaces.
 *
 * Returns SWA_OK or a negative swa_status_t (SWA_ERR_SHAPE for a bad base,
 * pairing flag, ring_W or a workspace that is too small).
 */
SWA_API size_t swa_sink_attn_fwd_rope_workspace(int total_tokens, int Hq, int Hkv, int D,
                                                int window);
SWA_API int swa_sink_attn_fwd_rope(const void *q, const void *k, const void *v,
                                   const int32_t *cu_seqlens, int num_seqs, int max_seqlen,
                                   int total_tokens, int Hq, int Hkv, int D, int window,
                                   const float *sink, float softmax_scale, float rope_base,
                                   int rope_interleaved, const int32_t *pos0, void *k_ring,
                                   void *v_ring, int ring_W, void *workspace,
                                   size_t workspace_bytes, void *o, float *lse, void *stream);

/*
 * Backward of swa_sink_attn_fwd: the gradients of q, k, v and of the sink for
 * an output gradient dout.
 *
 * Source: the forward of section 2.2.2 of the report summary above; the
 * pages give no backward (the ICML 2026 talk write-up's Q&A stresses that the
 * sink's initialisation and gradient updates must stay stable at scale). With
 * p_ij = exp(scale q_i.k_j - lse_i) over the visible keys and
 * p_sink,i = exp(s_h - lse_i):
 *   Delta_i = dout_i . o_i,   dS_ij = p_ij (dout_i . v_j - Delta_i)
 *   dq_i = scale sum_j dS_ij k_j,   dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i p_ij dout_i,       dsink_h = -sum_i p_sink,i Delta_i
 * with dk, dv of a kv head summed over its Hq/Hkv query heads.
 *
 *   q, k, v, cu_seqlens, num_seqs, max_seqlen, total_tokens, Hq, Hkv, D,
 *   window, sink, softmax_scale   as given to swa_sink_attn_fwd
 *   o, lse      the forward's outputs (bf16 [total, Hq, D], fp32 [Hq, total]);
 *               lse is required
 *   dout        bf16 [total, Hq, D]
 *   dq          bf16 [total, Hq, D] output; dk, dv bf16 [total, Hkv, D] outputs
 *   dsink       fp32 [Hq] output (zero without a sink), or NULL
 *   workspace   device memory of swa_sink_attn_bwd_workspace() bytes (Delta,
 *               fp32 [Hq, total]), 16-byte aligned, owned by the caller; calls
 *               that overlap in time need separate workspaces.
 *   Hq/Hkv must divide 64; D 64 or 128 (else SWA_ERR_UNSUPPORTED).
 *   dsink is zeroed and then accumulated on the stream (atomic adds: the
 *   order of its fp32 sums, and so its last bits, can differ between calls).
 *
 * Returns SWA_OK or a negative swa_status_t.
 */
SWA_API size_t swa_sink_attn_bwd_workspace(int total_tokens, int Hq);
SWA_API int swa_sink_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                              const void *dout, const float *lse, const int32_t *cu_seqlens,
                              int num_seqs, int max_seqlen, int total_tokens, int Hq, int Hkv,
                              int D, int window, const float *sink, float softmax_scale,
                              void *dq, void *dk, void *dv, float *dsink, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Decode / draft verification over a W-slot KV ring per sequence.
 *
 * Source: section 2.3 "Lightweight MTP" of the report summary above (draft
 * tokens from the MTP layers are verified by the main model in parallel,
 * raising arithmetic intensity without more KV-cache I/O), section 2.2.1
 * (SWA keeps a constant window of W tokens), and the Q&A of the ICML 2026
 * talk write-up (hzrcw.cc): positions keep increasing while the window slides.
 *
 * Sequence b has n_q new tokens at absolute positions pos[b] .. pos[b]+n_q-1
 * (1 real token + n_q-1 drafts). The ring holds the committed tokens at
 * positions pos[b]-W .. pos[b]-1, the token at position p in slot p mod W;
 * slots whose position would be negative are ignored. Query t sees the ring
 * tokens at positions >= pos[b]+t-W+1 and the new tokens 0..t (causal among
 * themselves). The ring is read-only here (see swa_sink_kv_commit).
 *
 *   q             bf16 [B, n_q, Hq, D]
 *   k_new, v_new  bf16 [B, n_q, Hkv, D]   keys/values of the new tokens
 *   k_ring,v_ring bf16 [B, W, Hkv, D]
 *   pos           int32 [B] device, >= 0 (a negative entry is treated as 0
 *                 and flagged)
 *   n_q           1..8;  W: 1..256;  D: 64 or 128;  n_q*(Hq/Hkv) <= 32.
 *   sink, softmax_scale  as for swa_sink_attn_fwd.
 *   o             bf16 [B, n_q, Hq, D]
 *   lse           fp32 [B, n_q, Hq] (natural log), or NULL.
 */
SWA_API int swa_sink_attn_decode(const void *q, const void *k_new, const void *v_new,
                         const void *k_ring, const void *v_ring,
                         const int32_t *pos, int B, int n_q, int Hq, int Hkv,
                         int D, int W, const float *sink, float softmax_scale,
                         void *o, float *lse, void *stream);

/*
 * Decode / draft verification over a long KV cache, split over the cached
 * positions: the global-attention layers of section 2.2 of the report summary
 * above (every earlier token visible) at decode, with the MTP verification of
 * section 2.3 and the sink of section 2.2.2.
 *
 * The cache follows the ring convention of swa_sink_attn_decode (the token at
 * position p in slot p mod W; query t sees cached positions
 * max(0, pos[b]+t-W+1) .. pos[b]-1 and the new tokens 0..t), so the result is
 * exactly what swa_sink_attn_decode defines, for any W that is a multiple of
 * 64. With W at least the context length the cache is a plain array indexed
 * by position and every earlier token is visible (a global layer).
 *
 *   k_cache, v_cache  bf16 [B, W, Hkv, D]
 *   max_ctx   an upper bound on every pos[b] (the host does not read pos): it
 *             sizes the split. A pos[b] beyond the cover is flagged (bit 1 of
 *             swa_sink_device_error) and its excess positions are skipped.
 *   workspace device memory of at least swa_sink_decode_splitkv_workspace()
 *             bytes, 16-byte aligned, owned by the caller; it holds the
 *             partial softmax states between the two kernels of a call, so
 *             calls that overlap in time need separate workspaces.
 *   the other arguments as for swa_sink_attn_decode (n_q 1..8,
 *   n_q*(Hq/Hkv) <= 32, D 64 or 128).
 *
 * Returns SWA_OK or a negative swa_status_t (SWA_ERR_UNSUPPORTED when W is
 * not a multiple of 64; SWA_ERR_SHAPE when the workspace is too small).
 */
SWA_API size_t swa_sink_decode_splitkv_workspace(int B, int n_q, int Hq, int Hkv, int D,
                                                 int W, int max_ctx);
SWA_API int swa_sink_attn_decode_splitkv(const void *q, const void *k_new, const void *v_new,
                                         const void *k_cache, const void *v_cache,
                                         const int32_t *pos, int B, int n_q, int Hq, int Hkv,
                                         int D, int W, int max_ctx, const float *sink,
                                         float softmax_scale, void *o, float *lse,
                                         void *workspace, size_t workspace_bytes,
                                         void *stream);

/*
 * Commit accepted tokens into the ring after verification: for
 * u < n_accept[b], new token u (absolute position pos[b]+u) is copied into
 * slot (pos[b]+u) mod W of k_ring / v_ring. pos is not modified; the caller
 * advances it by n_accept. An n_accept[b] outside [0, n_q] is clamped and
 * flagged. Source: section 2.3 of the report summary above (only verified
 * draft tokens become part of the sequence).
 *
 *   k_ring, v_ring bf16 [B, W, Hkv, D] (updated in place)
 *   k_new, v_new   bf16 [B, n_q, Hkv, D]
 *   pos, n_accept  int32 [B] device
 */
SWA_API int swa_sink_kv_commit(void *k_ring, void *v_ring, const void *k_new,
                       const void *v_new, const int32_t *pos,
                       const int32_t *n_accept, int B, int n_q, int Hkv, int D,
                       int W, void *stream);

/*
 * Decode / draft verification and commit over an FP8 (E4M3) ring.
 *
 * Source: the KV cache of these models is sized as an FP8 cache (MiMo-V3 /
 * HySparse2 news page, hao.cnyes.com, cost comparison at one million tokens),
 * and inference runs in FP8 with the E4M3 format (MiMo-V2 blog review,
 * kokolerk.github.io, sections 4.3 and 6). No page fixes the scale
 * granularity; here it is one fp32 scale per kv head for K and one for V.
 *
 * The ring holds E4M3 codes (OCP E4M3FN: bias 7, no infinities, 0x7F / 0xFF
 * NaN, largest finite 448): the ring value of code c of kv head g is
 * value(c) * kv_scale[g] for K and value(c) * kv_scale[Hkv + g] for V. The
 * decode is then exactly swa_sink_attn_decode over those values (positions,
 * visibility, sink and outputs as there; the new tokens stay bf16).
 *
 *   k_ring, v_ring  uint8 E4M3 codes [B, W, Hkv, D], 16-byte aligned
 *   kv_scale        fp32 [2 * Hkv] device: K scales, then V scales; each
 *                   must be finite and > 0 (else flagged: bit 1 of
 *                   swa_sink_device_error, results undefined)
 *   the other arguments and limits as for swa_sink_attn_decode.
 *
 * swa_sink_kv_commit_fp8 writes accepted new token u (u < n_accept[b]) into
 * slot (pos[b]+u) mod W as the E4M3 codes of x / scale: the quotient rounded
 * to fp32 (IEEE division), then to the nearest E4M3 value (ties to even),
 * magnitudes beyond 448 saturated to 448 (NaN stays NaN). n_accept and pos
 * as for swa_sink_kv_commit.
 */
SWA_API int swa_sink_attn_decode_fp8kv(const void *q, const void *k_new, const void *v_new,
                                       const void *k_ring, const void *v_ring,
                                       const float *kv_scale, const int32_t *pos, int B,
                                       int n_q, int Hq, int Hkv, int D, int W,
                                       const float *sink, float softmax_scale, void *o,
                                       float *lse, void *stream);
SWA_API int swa_sink_kv_commit_fp8(void *k_ring, void *v_ring, const void *k_new,
                                   const void *v_new, const float *kv_scale,
                                   const int32_t *pos, const int32_t *n_accept, int B,
                                   int n_q, int Hkv, int D, int W, void *stream);

/* Human-readable text for a swa_status_t (static storage). */
SWA_API const char *swa_sink_status_string(int status);

/*
 * Device-side error flags recorded by kernels on the CURRENT device since the
 * last clear: bit 0 = a wait timed out, bit 1 = a device-resident argument
 * was out of range. Synchronises the device. *flags receives the bits; if
 * clear != 0 they are reset. Returns SWA_OK or SWA_ERR_CUDA.
 */
SWA_API int swa_sink_device_error(unsigned int *flags, int clear);

/* Library ABI version (major * 100 + minor). */
SWA_API int swa_sink_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_SINK_H */
