/*
 * ssd_i8.h -- C ABI of the B200 (sm_100a) int8-input Mamba-2 SSD library.
 *
 * The operation (per batch b and head h, head h reading group g = h / (nheads/ngroups)):
 *
 *   x_t = s_x[h] * xq[b,t,h,:]     B_t = s_B[g] * Bq[b,t,g,:]     C_t = s_C[g] * Cq[b,t,g,:]
 *   h_t = exp(dt_t * A[h]) * h_{t-1} + dt_t * x_t B_t^T            (state [headdim, dstate])
 *   y_t = h_t C_t + D[h] * x_t                                      (output [headdim])
 *
 * Sources: the SSM recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t ("Ternary Mamba: Grouped
 * Quantization-Aware Training of W1.58A16 State Space Models", section 1); x, B and C as
 * int8 SSD inputs with static scales ("Quamba2" OpenReview rebuttal, response on quantizing
 * the SSD inputs (B, C, x); "Quamba" project page, static per-tensor quantization; "SSDi8"
 * page, Table 10, per-H(G) scale axes); the chunked evaluation with a persistent int8 path
 * ("SSDi8" page, Abstract, Figure 1(b), Figure 3(a) ChunkState, Table 5 ChunkBMM).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; tensors are dense,
 *     row-major (C order) with the shapes given in brackets.  The library allocates nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Argument errors are detected on the host and returned before anything is launched;
 *     launch failures return SSD_ERR_CUDA.  No entry point throws or aborts.
 *   - Output dtype codes: SSD_OUT_F32 (float), SSD_OUT_F16 (IEEE half), SSD_OUT_I8 (int8,
 *     q = clamp(round_half_even(y * fp32(1 / y_scale)), -127, 127), the product taken exactly
 *     and rounded once; y_scale > 0 is used only for I8).
 */
#ifndef SSD_I8_H
#define SSD_I8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1, /* null pointer, negative size, H % G != 0, bad dtype code ... */
    SSD_ERR_UNSUPPORTED = 2, /* shape outside what the kernels implement (see each call)   */
    SSD_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned                  */
    SSD_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed                 */
    SSD_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up (reported by a kernel)   */
} ssd_status;

typedef enum ssd_out_dtype { SSD_OUT_F32 = 0, SSD_OUT_F16 = 1, SSD_OUT_I8 = 2 } ssd_out_dtype;

/*
 * Flag OR-ed into the y_dtype of ssd_i8_chunk_scan / _varlen / _noalloc and of the decode steps
 * ssd_i8_state_update / _q8: the output is y' = H y / 8 per (token, head) over the 64 head
 * channels (H the 64 x 64 Hadamard matrix in
 * Sylvester order, H[q][p] = (-1)^popcount(p & q), so y' is an orthonormal transform of y),
 * applied before the conversion to y_dtype -- the Hadamard transform of the SSD output ahead of
 * out_proj that the Quamba2 OpenReview rebuttal uses with its Table R10 runs, fused into the
 * kernel's epilogue.  For SSD_OUT_I8, y_scale quantises y'.  Requires headdim 64 (else
 * SSD_ERR_UNSUPPORTED).  The states are not affected.
 */
#define SSD_OUT_HADAMARD 16

/*
 * Flag OR-ed into the y_dtype of ssd_i8_chunk_scan / _varlen / _noalloc and of the decode steps
 * ssd_i8_state_update / _q8: B_scale and C_scale are per group AND dstate channel, float
 * [ngroups, dstate] (row-major), instead of per group -- the per-P(N) quantization axis of the
 * SSDi8 page, Table 10: B_t[n] = s_B[g, n] Bq[t, g, n] and C_t[n] = s_C[g, n] Cq[t, g, n].  In
 * the chunk scan the products s_C[g, n] s_B[g, n] then sit inside ChunkBMM, which runs on f16
 * tensor cores (Cq exact, Bq s_C s_B / max_n(s_C s_B) rounded to f16) instead of exact int8;
 * the chunk state and C H take the channel scales exactly.  The states (init_state,
 * final_state, the cached decode state) are the true states, as without the flag.
 */
#define SSD_SCALES_PER_N 32

/* Version of this ABI; bumped when a signature or a layout changes. */
SSD_API int ssd_i8_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
SSD_API const char *ssd_status_string(ssd_status status);

/*
 * Bytes of device workspace that ssd_i8_chunk_scan needs for this problem (0 on invalid
 * sizes): a status word, hand-off flags and one 32 KiB state slot per CTA of the persistent
 * kernel (at most 256 CTAs, so at most about 8.4 MB).  Its contents need no initialisation:
 * every flag and the status word are tagged with a per-call 64-bit epoch.  One workspace per
 * concurrently running call.
 */
SSD_API size_t ssd_i8_chunk_scan_workspace_size(int batch, int seqlen, int nheads, int headdim,
                                        int dstate, int ngroups, int chunk_size);

/*
 * Chunked SSD scan over a prefill (SSDi8 page: ChunkState, state passing, ChunkScan with the
 * ChunkBMM product CB = C B^T kept in exact int32).
 *
 *   x          int8  [batch, seqlen, nheads, headdim]
 *   B, C       int8  [batch, seqlen, ngroups, dstate]
 *   dt         float [batch, seqlen, nheads]   (already discretised / softplus'ed, >= 0)
 *   A, D       float [nheads]                   (A <= 0)
 *   x_scale    float [nheads];  B_scale, C_scale float [ngroups]   (static scales; float
 *              [ngroups, dstate] with SSD_SCALES_PER_N in y_dtype)
 *   chunk_size Q: 64, 128 or 256.  The result does not depend on Q beyond rounding.
 *   init_state float [batch, nheads, headdim, dstate] or NULL (zero initial state)
 *   final_state float [batch, nheads, headdim, dstate] or NULL (not written)
 *   y          [batch, seqlen, nheads, headdim] of y_dtype (an SSD_OUT_* code, optionally
 *              OR-ed with SSD_OUT_HADAMARD and SSD_SCALES_PER_N)
 *   workspace  device memory of at least ssd_i8_chunk_scan_workspace_size(...) bytes,
 *              256-byte aligned.
 * Supported: headdim == 64; dstate in {16, 32, 64, 128}; batch * nheads < 2^31 (larger:
 * SSD_ERR_UNSUPPORTED); seqlen >= 0 (seqlen == 0 only copies
 * init_state to final_state); batch >= 0; nheads % ngroups == 0; x, B, C and y 16-byte
 * aligned.  Expected ranges: A <= 0 and dt >= 0 (a decaying state); other values are computed
 * but without the range guarantees the f16 operand scaling relies on.
 * Device-side failures (a bounded wait that gave up) do not change the return value of this
 * asynchronous call; ssd_i8_chunk_scan_status reports them.
 */
SSD_API ssd_status ssd_i8_chunk_scan(const int8_t *x, const int8_t *B, const int8_t *C, const float *dt,
                             const float *A, const float *D, const float *x_scale,
                             const float *B_scale, const float *C_scale, int batch, int seqlen,
                             int nheads, int headdim, int dstate, int ngroups, int chunk_size,
                             const float *init_state, float *final_state, void *y, int y_dtype,
                             float y_scale, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Workspace bytes of ssd_i8_chunk_scan_varlen for `nseq` sequences (about 8.4 MB plus 16 bytes
 * per sequence); 0 for nseq < 0.
 */
SSD_API size_t ssd_i8_chunk_scan_varlen_workspace_size(int nseq);

/*
 * Chunked SSD scan over packed variable-length sequences and strided inputs: the same
 * computation as ssd_i8_chunk_scan, with the state starting afresh (from init_state[s] or zero)
 * at the first token of every sequence s.  This is the prefill of a serving batch whose prompts
 * are packed back to back, reading x, B, C and dt straight out of a wider projection output.
 *
 *   cu_seqlens HOST int32 [nseq + 1]: sequence s is packed tokens [cu_seqlens[s],
 *              cu_seqlens[s + 1]); non-decreasing, inside [0, total_tokens].  Empty sequences
 *              are allowed (their final state is their initial state).  Tokens outside every
 *              sequence are read but never written.
 *   x          int8 rows of x_token_stride bytes, one per packed token; a row starts with the
 *              nheads x headdim values of that token (x_token_stride >= nheads * headdim, a
 *              multiple of 16).
 *   B, C       int8 rows of bc_token_stride bytes, each starting with ngroups x dstate values
 *              (bc_token_stride >= ngroups * dstate, a multiple of 16).
 *   dt         float rows of dt_token_stride elements starting with nheads values
 *              (dt_token_stride >= nheads).
 *   A, D, scales, chunk_size, y_dtype, y_scale: as for ssd_i8_chunk_scan.
 *   init_state float [nseq, nheads, headdim, dstate] or NULL; final_state likewise (not written
 *              if NULL).
 *   y          [total_tokens, nheads, headdim] of y_dtype, contiguous; rows of tokens outside
 *              every sequence are left untouched.
 *   workspace  at least ssd_i8_chunk_scan_varlen_workspace_size(nseq) bytes, 256-byte aligned.
 * The sequence table is uploaded with cudaMemcpyAsync from host memory on `stream` (staged
 * before the call returns), so the call cannot be captured into a CUDA graph.  Shapes, base
 * alignments and error reporting are those of ssd_i8_chunk_scan (with the non-empty sequences
 * in place of batch: their count times nheads < 2^31); SSD_ERR_INVALID_ARG also covers
 * malformed cu_seqlens and strides.
 */
SSD_API ssd_status ssd_i8_chunk_scan_varlen(const int8_t *x, long long x_token_stride,
                                            const int8_t *B, const int8_t *C,
                                            long long bc_token_stride, const float *dt,
                                            long long dt_token_stride, const float *A,
                                            const float *D, const float *x_scale,
                                            const float *B_scale, const float *C_scale,
                                            const int32_t *cu_seqlens, int nseq,
                                            long long total_tokens, int nheads, int headdim,
                                            int dstate, int ngroups, int chunk_size,
                                            const float *init_state, float *final_state, void *y,
                                            int y_dtype, float y_scale, void *workspace,
                                            size_t workspace_bytes, void *stream);

/*
 * Status of the chunk-scan calls (ssd_i8_chunk_scan or _varlen) that ran on `workspace` since
 * the previous status query on it (or, with none, since the first call): synchronises `stream`,
 * then returns SSD_ERR_TIMEOUT if a device-side wait of any of them gave up (a CTA waiting for
 * its predecessor's state hand-off, or for a tensor-core / TMA completion) and SSD_OK otherwise.
 * Every wait inside the kernels is bounded (about one second), so a failed call still
 * terminates; its outputs are then undefined.  Calls on one workspace are assumed to come from
 * one host thread at a time (they may not overlap anyway).
 */
SSD_API ssd_status ssd_i8_chunk_scan_status(const void *workspace, void *stream);

/*
 * Test hook for failure detection (not for production use).  Arms a one-shot fault for the next
 * ssd_i8_chunk_scan launch in this process: the CTA with index `drop_publish_cta` skips publishing
 * its state hand-off (so its successor's bounded wait runs out), and every device-side wait of
 * that launch is bounded by `wait_cycles` SM clocks (<= 0 keeps the default of about one second).
 * The launch still terminates; ssd_i8_chunk_scan_status then reports SSD_ERR_TIMEOUT and later
 * calls run normally.  drop_publish_cta = -1 only shortens the waits.
 */
SSD_API ssd_status ssd_i8_debug_inject(int drop_publish_cta, long long wait_cycles);

/*
 * Allocation-free variant of ssd_i8_chunk_scan.  The pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory when they run the scan -- code working
 * inside a memory pool reserved in full up front, code that must not risk the device
 * synchronisation a cudaMalloc can cause, or a plug-in whose host owns every allocation.
 *
 * Arguments, supported shapes and results are those of ssd_i8_chunk_scan without the workspace:
 * the scratch comes from one array of 4 MiB compiled into the library as device memory, which
 * every GPU that loads the library holds until the process exits.  The call allocates nothing
 * (no cudaMalloc / cudaFree, no allocating library routine).
 *   - Size limit: problems whose ssd_i8_chunk_scan_workspace_size(...) exceeds 4 MiB
 *     (4194304 bytes) are rejected with SSD_ERR_WORKSPACE before anything is launched.  The
 *     kernel works in blocks of 128 tokens whatever chunk_size is, and that size counts them:
 *     the limit is batch * nheads * ceil(seqlen / 128) <= 127.
 *   - Device: the scratch of the device that is current at the call is used; `stream` must
 *     belong to that device.  The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it; make that first call before any stream capture.
 *   - Sharing: all calls on a device share the one array and it keeps the last call's
 *     contents.  Nothing in it needs to start at zero (its flags carry a per-call epoch), but
 *     calls whose execution overlaps on the GPU -- on different streams, or from different
 *     host threads -- race on it and give wrong results; serialise them (one stream, or
 *     events).
 */
SSD_API ssd_status ssd_i8_chunk_scan_noalloc(const int8_t *x, const int8_t *B, const int8_t *C,
                                             const float *dt, const float *A, const float *D,
                                             const float *x_scale, const float *B_scale,
                                             const float *C_scale, int batch, int seqlen,
                                             int nheads, int headdim, int dstate, int ngroups,
                                             int chunk_size, const float *init_state,
                                             float *final_state, void *y, int y_dtype,
                                             float y_scale, void *stream);

/*
 * Status of the ssd_i8_chunk_scan_noalloc calls on the current device since the previous query
 * -- the counterpart of ssd_i8_chunk_scan_status for callers that have no workspace to pass:
 * synchronises `stream`, then returns SSD_ERR_TIMEOUT if a device-side wait of one of them gave
 * up (its outputs are then undefined) and SSD_OK otherwise, also when no allocation-free call
 * has run on the device.  It reads the status words the kernel keeps at the start of the
 * built-in scratch.  Allocates nothing.
 */
SSD_API ssd_status ssd_i8_chunk_scan_noalloc_status(void *stream);

/*
 * Single-token decode state update, in place (the "SSD update" of the Quamba2 rebuttal's
 * generation-time discussion, Tables R7/R8): one step of the recurrence above.
 *
 *   state      float [batch, nheads, headdim, dstate]   read and overwritten with h_t
 *   x          int8  [batch, nheads, headdim]
 *   B, C       int8  [batch, ngroups, dstate]
 *   dt         float [batch, nheads]
 *   A, D, x_scale float [nheads]; B_scale, C_scale float [ngroups] ([ngroups, dstate] with
 *              SSD_SCALES_PER_N in y_dtype)
 *   y          [batch, nheads, headdim] of y_dtype
 * Supported: dstate in {16, 32, 64, 128, 256}; 1 <= headdim <= 256; nheads % ngroups == 0.
 */
SSD_API ssd_status ssd_i8_state_update(float *state, const int8_t *x, const int8_t *B, const int8_t *C,
                               const float *dt, const float *A, const float *D,
                               const float *x_scale, const float *B_scale, const float *C_scale,
                               int batch, int nheads, int headdim, int dstate, int ngroups,
                               void *y, int y_dtype, float y_scale, void *stream);

/*
 * int8 cached SSM state (the quantized cached states of the Quamba2 rebuttal's generation-time
 * discussion, Tables R7/R8): the state of one (batch, head) is kept as int8 codes with one fp32
 * scale, h = state_scale[b, h] * state_q[b, h, p, n], i.e. one byte per element instead of four.
 * Quantisation rule (used by both calls below): scale = max|h| / 127 over the (batch, head)
 * state, code = clamp(round_half_even(h / scale), -127, 127); an all-zero state gets scale 0.
 *
 * ssd_i8_state_quantize: fp32 state [batch, nheads, headdim, dstate] (for instance the
 * final_state of a prefill) -> state_q int8 [same shape] and state_scale float [batch, nheads].
 */
SSD_API ssd_status ssd_i8_state_quantize(const float *state, int8_t *state_q, float *state_scale,
                                         int batch, int nheads, int headdim, int dstate,
                                         void *stream);

/*
 * One decode step on the int8 cached state, in place: dequantise, apply the step of
 * ssd_i8_state_update in fp32 (y from the updated fp32 state), then requantise with the rule
 * above (a fresh scale per step).  Arguments as for ssd_i8_state_update, with state_q /
 * state_scale in place of the fp32 state.
 * Supported: dstate in {16, 32, 64, 128, 256}; headdim * dstate <= 16384; nheads % ngroups == 0;
 * state_q, B and C 16-byte aligned.
 */
SSD_API ssd_status ssd_i8_state_update_q8(int8_t *state_q, float *state_scale, const int8_t *x,
                                          const int8_t *B, const int8_t *C, const float *dt,
                                          const float *A, const float *D, const float *x_scale,
                                          const float *B_scale, const float *C_scale, int batch,
                                          int nheads, int headdim, int dstate, int ngroups,
                                          void *y, int y_dtype, float y_scale, void *stream);

/*
 * ChunkBMM of SSDi8 (Table 5): the exact int32 products CB[b, c, g, t, s] =
 * sum_n Cq[b, c*Q+t, g, n] * Bq[b, c*Q+s, g, n] for every chunk c of length Q, the full
 * Q x Q block (no causal mask), zero where c*Q+t or c*Q+s >= seqlen.  Computed by the same
 * device code the chunk scan uses for its intra-chunk term; exposed so that the integer part
 * of the scan can be checked bit for bit.
 *
 *   C, B int8 [batch, seqlen, ngroups, dstate];  cb int32 [batch, ceil(seqlen/Q), ngroups, Q, Q]
 * Supported: as ssd_i8_chunk_scan for dstate and chunk_size.
 */
SSD_API ssd_status ssd_i8_chunk_cb(const int8_t *C, const int8_t *B, int batch, int seqlen, int ngroups,
                           int dstate, int chunk_size, int32_t *cb, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_I8_H */
