/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention library, libfa.so.
 *
 * The operation (page "Flash Attention — 長い系列を扱う Transformer の学習と推論を速くする", quick start and
 * Workflow 1 Step 2; page "FlashAttention（フラッシュアテンション）とは？…", sections "FlashAttentionの仕組み"
 * and "Online Softmax"): exact scaled dot-product attention
 *
 *     O = softmax(scale * Q K^T + causal mask) V
 *
 * computed tile by tile with an online softmax, so the Sq x Sk score matrix never reaches device memory, plus
 * the backward pass that recomputes the probabilities from the saved log-sum-exp ("tiling and recomputation",
 * refbase entity page "FlashAttention", section "Capability"; training support: the glossary page's
 * misconception 2).
 *
 * Conventions shared by every entry point
 *   - Layout [batch, seqlen, nheads, headdim] ("[batch, seqlen, nheads, headdim]" in the skill page's
 *     flash_attn_func examples), contiguous, row-major: element (b, s, h, d) sits at ((b*S + s)*H + h)*D + d.
 *     q, out, dout, dq: [B, Sq, H, D];  k, v, dk, dv: [B, Sk, H, D] ([B, Sk, Hkv, D] in the entry points
 *     that take Hkv);  lse: fp32 [B, H, Sq].
 *   - dtype: FA_F16 or FA_BF16 for every 16-bit tensor of a call (the pages: fp16/bf16 only, no fp32); the
 *     e4m3 forward (fa_fwd_fp8) takes 8-bit q, k, v and writes bf16.
 *   - D (head dim) in {64, 128}. B, H, Sq, Sk >= 1. Every pointer 16-byte aligned, device memory.
 *   - scale: 0.0f (or -0.0f) means 1/sqrt(D) (the pages' softmax_scale=None "Auto-scale"); any other finite value,
 *     negative ones included, is used as given; a non-finite scale is FA_ERR_INVALID.
 *   - causal != 0 applies the causal mask, bottom-right aligned when Sq != Sk: key j is visible to query i
 *     iff j <= i + (Sk - Sq). A query row that sees no key gets O = 0 and LSE = -inf.
 *   - lse[b,h,i] = ln sum_{j visible} exp(scale * q_i . k_j), fp32 (natural log, scale included).
 *   - Ownership: the caller allocates and owns every buffer, including the backward workspace. The library
 *     allocates no device memory; it keeps no per-call state besides a device-side sticky error word and a
 *     small host-side cache of encoded TMA descriptors (keyed by pointer and shape, so reusing a buffer is safe).
 *   - Asynchrony: all work is enqueued on `stream` (0 = legacy default stream). A return of FA_OK means the
 *     launches were accepted, not that they finished. A kernel that gives up on an internal wait (bounded
 *     spin, about 2 s) records FA_ERR_TIMEOUT in the device status word (fa_device_status) and exits cleanly.
 *   - Errors: invalid arguments return FA_ERR_INVALID and launch nothing; an unsupported head dim, dtype or
 *     device returns FA_ERR_UNSUPPORTED and launches nothing; a CUDA launch failure returns FA_ERR_CUDA.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t; /* identical to the CUDA runtime's definition */

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

typedef enum { FA_F16 = 0, FA_BF16 = 1 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = -1,     /* bad pointer, size, alignment, non-finite scale or dtype; nothing launched */
  FA_ERR_UNSUPPORTED = -2, /* head dim not in {64,128}, or the current device is not sm_100 */
  FA_ERR_CUDA = -3,        /* a CUDA call or kernel launch failed */
  FA_ERR_TIMEOUT = -4,     /* device status only: a kernel gave up on a bounded wait */
  FA_ERR_WORKSPACE = -5    /* backward workspace missing, misaligned or smaller than fa_bwd_workspace_size */
} fa_status;

/*
 * Forward: out = softmax(scale * q k^T [+ mask]) v and lse (see conventions above).
 *   q [B,Sq,H,D], k [B,Sk,H,D], v [B,Sk,H,D]: inputs, read only.
 *   out [B,Sq,H,D]: written, same dtype as the inputs.  lse [B,H,Sq] fp32: written.
 * Returns FA_OK or a negative fa_status.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H, int D,
           int causal, float scale, int dtype, cudaStream_t stream);

/*
 * Forward with grouped K/V heads and a sliding window (skill page "Flash Attention — …", Workflow 2 Step 3:
 * multi-query attention with fewer KV heads, and Steps 2-3: window_size=(left, right)).
 *   H query heads, Hkv K/V heads (H a multiple of Hkv; Hkv = 1 is multi-query): query head h reads K/V head
 *   h / (H / Hkv); k and v are [B, Sk, Hkv, D].
 *   window_left, window_right: with c = i + Sk - Sq the key aligned with query i, key j is visible iff
 *   (window_left < 0 or j >= c - window_left) and (window_right < 0 or j <= c + window_right), on top of the
 *   causal rule (which caps the right side at c). Negative = unbounded ((-1, -1) = no window).
 * fa_fwd(..., H, ...) is fa_fwd_ex(..., H, H, ..., -1, -1, ...). Other conventions as above; additionally
 * FA_ERR_INVALID if Hkv < 1 or H is not a multiple of Hkv.
 */
FA_API int fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                     int H, int Hkv, int D, int causal, int window_left, int window_right, float scale, int dtype,
                     cudaStream_t stream);

/*
 * Forward with attention dropout (the `dropout_p` argument of the skill page's flash_attn_func call, Workflow 2
 * Step 2; the pages name it only). Arguments as fa_fwd_ex, plus:
 *   dropout_p  drop probability, 0 <= dropout_p < 1; it is rounded to t / 256 with t = floor(256 p + 1/2), and
 *              t = 256 is rejected (FA_ERR_INVALID).
 *   seed       64-bit Philox4x32-10 key (low word, high word).
 *   offset     32-bit counter word 3, so that successive calls with one seed draw different masks.
 * Element (i, j) of head number bh = b * H + h is kept iff byte (j mod 4) of word (i mod 4) of
 * Philox4x32-10(counter = (i / 4, j / 4, bh, offset), key = seed) is >= t. O = (P o Z) V with Z = keep / (1 -
 * t / 256); LSE is that of the undropped scores, so fa_bwd_dropout with the same seed and offset regenerates the
 * mask. dropout_p = 0 gives exactly fa_fwd_ex.
 */
FA_API int fa_fwd_dropout(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                          int H, int Hkv, int D, int causal, int window_left, int window_right, float scale, int dtype,
                          float dropout_p, uint64_t seed, uint32_t offset, cudaStream_t stream);

/*
 * Forward on 8-bit inputs (the FP8 forward of the skill page's Workflow 3: "FP8 is a forward-only path, and the
 * input must be float8_e4m3fn"). q, k, v hold e4m3 bytes ([B,Sq,H,D] and [B,Sk,Hkv,D]); their real values are
 * the e4m3 values times q_descale, k_descale and v_descale (positive finite per-tensor factors; 1 for plain
 * e4m3 inputs). out is bf16 [B,Sq,H,D], lse fp32 [B,H,Sq]. The probabilities enter the P V product rounded to
 * e4m3 (round to nearest, saturating), so O carries up to 2^-4 relative error per probability term. D in
 * {64, 128} (FA_ERR_UNSUPPORTED otherwise). Heads, window and scale as in fa_fwd_ex.
 */
FA_API int fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk,
                      int H, int Hkv, int D, int causal, int window_left, int window_right, float scale,
                      float q_descale, float k_descale, float v_descale, cudaStream_t stream);

/*
 * Backward of fa_fwd_dropout: arguments as fa_bwd_ex plus the forward's dropout_p, seed and offset (the same
 * values, or the gradients are those of another mask). out must be the dropped output fa_fwd_dropout returned.
 */
FA_API int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* out, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int Hkv, int D,
                          int causal, int window_left, int window_right, float scale, int dtype, float dropout_p,
                          uint64_t seed, uint32_t offset, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes (0 on invalid sizes). The workspace holds the fp32
 * dQ accumulator and the per-row fp32 terms D_i = rowsum(dO_i * O_i) and LSE_i * log2(e).
 */
FA_API size_t fa_bwd_workspace_size(int B, int Sq, int H, int D);

/*
 * Backward: given the forward's inputs, its outputs out and lse, and the upstream gradient dout, writes
 * dq [B,Sq,H,D], dk [B,Sk,H,D] and dv [B,Sk,H,D] (same dtype as the inputs). P is recomputed from lse; the S x S
 * matrices never reach device memory.
 *   workspace: caller-owned device buffer of at least fa_bwd_workspace_size(B,Sq,H,D) bytes, 256-byte aligned;
 *              its contents on entry do not matter and are overwritten.
 * Returns FA_OK or a negative fa_status (FA_ERR_WORKSPACE for a missing or short workspace).
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
           void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int D, int causal, float scale, int dtype,
           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Backward with grouped K/V heads and a sliding window (same arguments and readings as fa_fwd_ex): dk and dv
 * are [B, Sk, Hkv, D], each K/V head's gradient summed over its group of query heads; dq is [B, Sq, H, D].
 * The workspace size is fa_bwd_workspace_size(B, Sq, H, D) with H the number of query heads.
 */
FA_API int fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int Hkv, int D,
                     int causal, int window_left, int window_right, float scale, int dtype, void* workspace,
                     size_t workspace_bytes, cudaStream_t stream);

/*
 * The three launches of fa_bwd one at a time, for callers that time or schedule them separately:
 *   stage 0: D_i = rowsum(dO_i * O_i) and LSE_i * log2(e) into the workspace, and zero its dQ accumulator;
 *   stage 1: the main kernel (recomputes P per 128-key tile, writes dK and dV, accumulates dQ in fp32);
 *   stage 2: dq = dtype(scale * dQ accumulator).
 * Stages 0, 1, 2 in that order on one stream with identical arguments are exactly fa_bwd; stage -1 runs all
 * three. Arguments, validation and return codes are those of fa_bwd (an unknown stage is FA_ERR_INVALID).
 */
FA_API int fa_bwd_stage(int stage, const void* q, const void* k, const void* v, const void* out, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int D,
                        int causal, float scale, int dtype, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * Size of the fixed device scratch that fa_bwd_noalloc uses in place of a caller workspace (64 MiB).
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * fa_bwd without a workspace argument and without any device allocation, for callers that cannot call
 * cudaMalloc: for example a caller living inside another framework that owns every byte of device memory
 * and forbids allocations outside its own pool, or a latency-critical caller that cannot afford the
 * device-wide synchronisation cudaMalloc may cause. (The pages describe no such entry point; it is a
 * convenience of this library.)
 *   - The scratch is one statically sized array in the library's device image, FA_NOALLOC_SCRATCH_BYTES
 *     long. Every GPU that loads the library holds it until the process exits.
 *   - Problems whose fa_bwd_workspace_size exceeds FA_NOALLOC_SCRATCH_BYTES are rejected with
 *     FA_ERR_WORKSPACE before anything is launched (use fa_bwd with your own workspace for those).
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress) with that
 *     device current; make that first call before any stream capture on the device.
 *   - Every call shares the one array and it keeps the previous call's contents; the kernels clear what
 *     must start at zero themselves. Calls whose kernels overlap on the GPU (two streams, or two host
 *     threads) race on the array and give wrong gradients: serialise them.
 * Other arguments, outputs and return codes are those of fa_bwd.
 */
FA_API int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int D,
                          int causal, float scale, int dtype, cudaStream_t stream);

/* Static English description of a status code (never NULL). */
FA_API const char* fa_status_string(int status);

/*
 * Device-side sticky status word of the current device: FA_OK, or FA_ERR_TIMEOUT once a kernel gave up on a
 * bounded wait. Synchronises the device. With reset != 0 the word is cleared after reading. Returns the
 * status, or FA_ERR_CUDA if it could not be read.
 */
FA_API int fa_device_status(int reset);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
