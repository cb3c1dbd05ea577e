/*
 * glq.h -- C ABI of glq-b200, a B200 (sm_100a) library for GLQ's fused
 * compressed-weight linear layer
 *
 *     y = S_out . H_m . W^ . H_n . (S_in . x)
 *
 * Definitions (GLQ project pages):
 *   - glq 0.5.1 PyPI page, "How it works" 1: each 8-weight group of W^ is a
 *     16-bit index into a 65,536-entry E8 lattice codebook (the first shells
 *     of E8); 3-8 bpw add 8-bit (256-entry) or 16-bit (E8) residual stages.
 *   - same page, "How it works" 2: the Randomized Hadamard Transform is a
 *     random sign flip followed by a fast Walsh-Hadamard transform.
 *   - same page, "Bit widths": one global scale per layer; a size that is not
 *     a power of two uses a block-diagonal Hadamard over its binary
 *     decomposition (2688 = 2048 + 512 + 128).
 *   - same page, "Inference kernels": Y = X . dequant(W)^T computed against
 *     the indices without materialising W; residual index, residual codebook
 *     and inverse residual scale are arguments of the matmul.
 *   - GLQ v0.3.2 release notes, "What changed": the linear path is the three
 *     ops input_rht -> fused linear -> output_rht.
 *
 * Conventions fixed by this library where the pages leave them open:
 *   - codeword of group g in row r covers input columns 8g..8g+7; index
 *     arrays are row-major [m][n/8];
 *   - w^[r][8g+j] = ws * (cb1[idx1][j] + rs * cb2[idx2][j]) where rs is the
 *     multiplier applied at decode (the pages' inverse residual scale); from
 *     5 bpw every residual stage k adds rs_k * cb_k[idx_k][j], in the order
 *     of the "Bit widths" table (16-bit E8 stages, then the 8-bit stage);
 *   - H_k[i][j] = (-1)^popcount(i & j) / sqrt(k) per block, blocks of the
 *     binary decomposition of n in descending size at increasing offsets;
 *   - input side: sign then H_n; output side: H_m then sign.
 *
 * Threading and ordering: every call that takes a cudaStream_t is
 * asynchronous and stream-ordered.  The transient device buffers of
 * glq_linear (rotated activations, split-K partial sums, pre-rotation
 * outputs, the reconstructed fp16 W of large batches) live in one workspace
 * per device shared by all its layers, so the glq_linear calls of one device
 * must be serialised on the GPU (one stream, or explicit events).  A layer
 * itself owns only its indices, signs and a few counter words.  Handles are
 * not thread-safe.  Every function returns a status and never throws.
 */
#ifndef GLQ_B200_H
#define GLQ_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GLQ_API __attribute__((visibility("default")))
#else
#define GLQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GLQ_OK = 0,
    GLQ_ERR_INVALID_ARG = 1,  /* null pointer, bad sign value, bad scale */
    GLQ_ERR_SHAPE = 2,        /* m, n not positive multiples of 8; B < 0; size limits */
    GLQ_ERR_DTYPE = 3,        /* unsupported dtype combination */
    GLQ_ERR_BPW = 4,          /* bpw not in 2..8 or inconsistent residual stages */
    GLQ_ERR_NO_CODEBOOK = 5,  /* missing or wrong-sized codebook handle */
    GLQ_ERR_OOM = 6,          /* device or host allocation failed */
    GLQ_ERR_CUDA = 7,         /* a CUDA runtime call or launch failed */
    GLQ_ERR_DEVICE_CHECK = 8, /* a device-side check recorded a fault */
    GLQ_ERR_TIMEOUT = 9,      /* a bounded device-side wait gave up */
    GLQ_ERR_UNSUPPORTED = 10, /* codebook contents the kernels cannot hold */
    GLQ_ERR_CAPTURE = 11      /* the call needs a larger device workspace while its
                                 stream is being captured: reserve first */
} glq_status;

typedef enum { GLQ_F16 = 0, GLQ_BF16 = 1, GLQ_F32 = 2 } glq_dtype;

/* Opaque handles; `void*` stream arguments are cudaStream_t (0 = legacy). */
typedef struct glq_codebook_s *glq_codebook;
typedef struct glq_layer_s *glq_layer;

/* Human-readable name of a status.  Never NULL; static storage. */
GLQ_API const char *glq_status_str(glq_status s);

/* Library version string, static storage. */
GLQ_API const char *glq_version(void);

/*
 * glq_e8_codebook -- the library's E8 shell codebook (host only, no GPU).
 * Definition: glq 0.5.1 PyPI page, "How it works" 1 ("65,536 vectors from
 * the first seven shells of the E8 lattice").  The subset is fixed by this
 * library: every E8 point x (all coordinates integers, or all integers plus
 * 1/2, with an even coordinate sum) of squared norm <= 12, sorted by
 * (squared norm, x0, x1, ..., x7) ascending, first 65,536 kept.
 * out_fp16_bits: caller-owned host array of 65536*8 uint16 receiving the
 * IEEE binary16 bit patterns, row-major [65536][8] (every value is exact).
 * Errors: GLQ_ERR_INVALID_ARG if out_fp16_bits is NULL.
 */
GLQ_API glq_status glq_e8_codebook(uint16_t *out_fp16_bits);

/*
 * glq_codebook_upload -- copy a codebook to the current CUDA device.
 * Definition: glq 0.5.1 PyPI page, "How it works" 1 and "Bit widths".
 * host_fp16_bits: caller-owned host array [entries][dim] of fp16 bit
 *   patterns, read during the call only.
 * entries: 65536 (a 16-bit primary / residual table) or 256 (an 8-bit
 *   residual table); dim must be 8.
 * A 65,536-entry table must hold values k/2 with |k| <= 6 whose
 *   negation-folded size fits the on-chip table (true for glq_e8_codebook's
 *   table); otherwise GLQ_ERR_UNSUPPORTED.  A 256-entry table may hold any
 *   finite fp16 values.
 * out: receives a library-owned handle; release with glq_codebook_destroy
 *   after every layer that uses it has been destroyed.
 * Errors: GLQ_ERR_INVALID_ARG (NULL pointers, non-finite values),
 *   GLQ_ERR_SHAPE (entries/dim), GLQ_ERR_UNSUPPORTED, GLQ_ERR_OOM,
 *   GLQ_ERR_CUDA.  Synchronous.
 */
GLQ_API glq_status glq_codebook_upload(const uint16_t *host_fp16_bits, int32_t entries, int32_t dim,
                               glq_codebook *out);
GLQ_API glq_status glq_codebook_destroy(glq_codebook cb);

/*
 * glq_layer_create -- build a compressed linear layer on the current device.
 * Definition: glq 0.5.1 PyPI page, "How it works" 1-2, "Bit widths",
 * "Inference kernels" (Qidxs, Qidxs2, codebook2, Wscale, inv_resid_scale).
 * m, n: output / input features, positive multiples of 8, each <= 32768
 *   (the largest Hadamard row the one-CTA-per-row transforms hold).
 * bpw: 2 (primary only), 3 (primary + uint8 residual into a 256-entry
 *   table) or 4 (primary + uint16 residual into the E8 table).
 * idx1: host uint16 [m][n/8]; idx2: host uint8 [m][n/8] (bpw 3), host
 *   uint16 [m][n/8] (bpw 4) or NULL (bpw 2).  Both are read during the call
 *   only (copied and re-laid-out for the kernels).
 * primary: a 65,536-entry codebook handle.  residual: a 256-entry handle
 *   for bpw 3; for bpw 4 NULL or the primary handle itself (the E8 table);
 *   NULL for bpw 2.
 * weight_scale: ws, finite.  resid_scale: rs, finite (ignored for bpw 2).
 * s_in [n], s_out [m]: host int8, every entry +1 or -1.
 * out: receives the layer handle (library-owned; glq_layer_destroy).
 * Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_SHAPE, GLQ_ERR_BPW,
 *   GLQ_ERR_NO_CODEBOOK, GLQ_ERR_OOM, GLQ_ERR_CUDA.  Synchronous.
 */
GLQ_API glq_status glq_layer_create(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1,
                            const void *idx2, glq_codebook primary, glq_codebook residual,
                            float weight_scale, float resid_scale, const int8_t *s_in,
                            const int8_t *s_out, glq_layer *out);

/*
 * glq_layer_create_stages -- glq_layer_create for every bit width of the
 * "Bit widths" table on the glq 0.5.1 PyPI page: bpw 2..8 is a 16-bit
 * primary E8 index per 8 weights followed by (bpw - 2) / 2 residual stages of
 * 16-bit E8 indices and, for an odd bpw, one last stage of 8-bit indices
 * into a 256-entry table (5 = 16+16+8, 6 = 16+16+16, 7 = 16+16+16+8,
 * 8 = 16+16+16+16).  Mixed-precision models are layers of different bpw.
 * w^[r][8g+j] = ws * c with c = cb1[idx1][j], then for each residual stage k
 *   in that order c = fma_f32(rs_k, cb_k[idx_k][j], c).
 * idx_res: host array of pointers, one per residual stage in stage order:
 *   uint16 [m][n/8] for a 16-bit stage, uint8 [m][n/8] for the 8-bit stage
 *   (may be NULL for bpw 2).  Read during the call only.
 * resid_scales: host float per residual stage (same order), finite.
 * residual: the 256-entry codebook for an odd bpw; otherwise NULL or the
 *   primary handle (16-bit stages index the E8 table).
 * Tensor-core calls (B > 16) of a layer above 4 bpw always reconstruct W in
 *   fp16 first (one fp16 fma per stage).
 * Other arguments, ownership and errors as glq_layer_create.  Synchronous.
 */
GLQ_API glq_status glq_layer_create_stages(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1,
                                           const void *const *idx_res, glq_codebook primary,
                                           glq_codebook residual, float weight_scale,
                                           const float *resid_scales, const int8_t *s_in,
                                           const int8_t *s_out, glq_layer *out);
GLQ_API glq_status glq_layer_destroy(glq_layer layer);

/*
 * glq_layer_create_shard -- the part of a layer that one GPU holds when the
 * layer is split over its input columns (row-parallel: y = sum over parts
 * of S_out . H_m . W^[:, part] . (H_n (S_in . x))[part], because H_m and
 * S_out are linear).  Arguments as glq_layer_create_stages, with the whole
 * layer's host arrays (idx1 and every idx_res [m][n/8], s_in [n], s_out [m]);
 * the shard keeps input columns [k_begin, k_end): k_begin a multiple of
 * 128, k_end a multiple of 128 or n.  Every GPU rotates the whole input x (x
 * is replicated) and computes its part's fp32 output; one all-reduce (sum)
 * of the parts' y over the GPUs, then glq_cast to the caller's dtype, gives
 * the layer's y.  glq_linear on a shard requires y_dtype == GLQ_F32; the
 * fused transforms, the batch-invariant mode and glq_linear_noalloc are not
 * available for shards.  glq_dequant_reference writes the shard's columns,
 * w_dev [m][k_end - k_begin].  Errors as glq_layer_create, GLQ_ERR_SHAPE for
 * a bad column range.  Synchronous.
 */
GLQ_API glq_status glq_layer_create_shard(int64_t m, int64_t n, int32_t bpw, const uint16_t *idx1,
                                          const void *const *idx_res, glq_codebook primary,
                                          glq_codebook residual, float weight_scale,
                                          const float *resid_scales, const int8_t *s_in, const int8_t *s_out,
                                          int64_t k_begin, int64_t k_end, glq_layer *out);

/*
 * glq_cast -- dst[i] = src[i] rounded to nearest even in `dtype`
 * (GLQ_F16, GLQ_BF16 or GLQ_F32), i < count; src_dev fp32 and dst_dev on the
 * current device.  Rounds the all-reduced fp32 output of row-parallel shards
 * to the model's dtype.  Errors: GLQ_ERR_SHAPE, GLQ_ERR_DTYPE,
 * GLQ_ERR_INVALID_ARG, GLQ_ERR_CUDA.  Asynchronous.
 */
GLQ_API glq_status glq_cast(const float *src_dev, void *dst_dev, glq_dtype dtype, int64_t count, void *stream);

/*
 * glq_layer_reserve -- grow the device's shared workspace so that every
 * glq_linear call on this layer with B <= max_B (decode and tensor-core
 * batches alike) finds its buffers already there: such calls then allocate
 * nothing and never synchronise, so they may be captured in a CUDA graph.
 * Reserve every layer first, then capture.  Without a reservation glq_linear
 * grows the workspace on demand: that synchronises the device and frees the
 * previous buffers, so graphs captured before a growth must not be replayed
 * after it; a growth needed while the call's stream is being captured
 * returns GLQ_ERR_CAPTURE instead.  Synchronous.  Errors: GLQ_ERR_SHAPE,
 * GLQ_ERR_OOM, GLQ_ERR_CUDA.
 */
GLQ_API glq_status glq_layer_reserve(glq_layer layer, int64_t max_B);

/*
 * glq_workspace_info -- bytes of device memory the shared workspace of
 * `device` holds (every layer's calls on that device use it).  Host only.
 * Errors: GLQ_ERR_INVALID_ARG.
 */
GLQ_API glq_status glq_workspace_info(int32_t device, size_t *bytes);

/*
 * glq_workspace_release -- synchronise `device` and free its shared
 * workspace; the next call that needs it allocates it again.  No captured
 * graph that used it may be replayed afterwards.  Errors:
 * GLQ_ERR_INVALID_ARG, GLQ_ERR_CUDA.
 */
GLQ_API glq_status glq_workspace_release(int32_t device);

/*
 * glq_linear -- y = S_out . H_m . W^ . H_n . (S_in . x).
 * Definition: the layer formula above (glq 0.5.1 PyPI page, "How it works",
 * "Inference kernels"; GLQ v0.3.2 release notes, input_rht ->
 * fused_linear_block_diag -> output_rht).
 * x_dev: device [B][n] row-major, dtype x_dtype (GLQ_F16 or GLQ_BF16),
 *   16-byte aligned.
 * y_dev: device [B][m] row-major, dtype y_dtype (== x_dtype, or GLQ_F32),
 *   16-byte aligned.
 * B >= 0 (B == 0 is a no-op).  stream: cudaStream_t.
 * Paths: B <= 16 runs the decode path: input RHT, the codebook GEMV on the
 *   legacy warp MMA with an on-chip codebook, and output RHT, launched back
 *   to back with programmatic dependent launch; by default the input RHT is
 *   folded into the GEMV launch where that measured faster (see
 *   glq_layer_set_fusion, which also sets either fusion explicitly); B > 16
 *   runs the tensor-core path:
 *   input RHT, one pass that reconstructs W = cb1 + rs cb2 as an fp16 matrix
 *   in the device's shared workspace, a TMA-fed tcgen05/TMEM GEMM on it
 *   (or, when glq_layer_set_prefill_reconstruct raises the bound above B, a
 *   tcgen05 GEMM whose producer warps rebuild each W tile in shared memory,
 *   W never stored), then output RHT.  The GEMV accumulates exactly
 *   in integers (fp64 across splits); the tensor-core path accumulates in
 *   fp32.
 * Workspace: the device's shared workspace (see glq_layer_reserve); a call
 *   it already covers allocates nothing and does not synchronise.
 * Errors: GLQ_ERR_INVALID_ARG (null or misaligned pointer), GLQ_ERR_DTYPE,
 *   GLQ_ERR_SHAPE, GLQ_ERR_OOM (workspace growth), GLQ_ERR_CAPTURE (growth
 *   needed during stream capture), GLQ_ERR_CUDA (launch failure).
 *   Asynchronous.
 */
GLQ_API glq_status glq_linear(glq_layer layer, const void *x_dev, glq_dtype x_dtype, void *y_dev,
                      glq_dtype y_dtype, int64_t B, void *stream);

/*
 * glq_layer_set_fusion -- choose how decode calls (B <= 16) run their two
 * transforms.  flags is a bit set: GLQ_FUSE_INPUT fuses the input RHT into
 * the GEMV launch (each task rotates its own aligned column range of x)
 * whenever B times the largest Hadamard block of n is at most 32768 values
 * and the tasks' activations fit shared memory; GLQ_FUSE_OUTPUT lets the last band of each Hadamard block of m rotate that
 * block in the same launch when B times the largest block of m fits the
 * library's bound; a cleared bit runs that transform as its own kernel.  The
 * default (GLQ_FUSE_DEFAULT) is the setting measured fastest on B200: cluster
 * split-K on, the output RHT as its own kernel, and the input RHT fused only
 * for rows longer than 8192 whose tasks are short (one task per CTA, at most
 * 1024 columns and 4096 values of x per task).  With both bits
 * cleared, every token's output is bitwise independent of the batch size for
 * B <= 16; otherwise that holds among batch sizes that take the same path.
 * GLQ_SPLITK_CLUSTER lets the split-K partial sums of a band of rows be
 * added through the distributed shared memory of a thread-block cluster (the
 * band's splits) instead of a global workspace and a last-arriving CTA,
 * whenever every CTA has one task and the splits fit a cluster; the
 * summation order is the same, so the results are bitwise identical.
 * All settings are bitwise reproducible run to run ("Bit-exact
 * determinism", glq 0.5.1 PyPI page, "Inference kernels") and agree within
 * the parity bound.  Errors: GLQ_ERR_INVALID_ARG (unknown bits).
 */
#define GLQ_FUSE_INPUT 1
#define GLQ_FUSE_OUTPUT 2
#define GLQ_SPLITK_CLUSTER 4
#define GLQ_FUSE_DEFAULT (-1)
GLQ_API glq_status glq_layer_set_fusion(glq_layer layer, int32_t flags);

/*
 * glq_layer_set_batch_invariant -- enable (1) or disable (0, the default) a
 * mode in which every token's output is the same bits whatever the batch
 * size it arrives in and whichever path a batch of that size would take
 * otherwise (the pages' claim that a prompt gives identical logits at B = 1
 * decode and in a batched prefill: glq 0.5.1 PyPI page, "Inference kernels",
 * "Bit-exact determinism").  In this mode every call, prefill-sized ones
 * included, runs the exact decode arithmetic: the input transform over all
 * tokens (the kernel chosen by n alone), the codebook GEMV on slices of at
 * most 16 tokens with one split plan per layer that no batch size changes
 * (integer sums of the E8 stages are exact; the fp32 sums of an 8-bit stage
 * then follow one order), and the output transform over all tokens (the
 * kernel chosen by m alone).  Batches above 16 tokens then run at GEMV speed
 * (the indices are read once per 16 tokens) instead of on the tensor cores.
 * Errors: GLQ_ERR_INVALID_ARG.
 */
GLQ_API glq_status glq_layer_set_batch_invariant(glq_layer layer, int32_t enable);

/*
 * glq_layer_set_prefill_reconstruct -- how tensor-core calls (B > 16) get
 * their weights.  Calls with B >= min_batch first reconstruct W = cb1 + rs
 * cb2 into an fp16 matrix of m_pad x n_pad (2 bytes per weight, in the
 * device's shared workspace: one such matrix, of the largest layer that
 * used it, per device) and run the TMA-fed tcgen05 GEMM on it; smaller
 * batches rebuild each W tile in shared memory inside the GEMM and never
 * materialise W (the pages' design: "Inference kernels", glq 0.5.1 PyPI
 * page).  Reconstructing once costs one pass over the indices, while the
 * dequantising producer repeats its codeword gathers for every 512 tokens;
 * measured on B200 the reconstruction is faster at every batch from 17
 * tokens, so the default (min_batch < 0) is 17: every tensor-core call
 * reconstructs.  A bound above a batch selects the producer for it (2-4 bpw;
 * layers above 4 bpw always reconstruct).  Errors: GLQ_ERR_INVALID_ARG.
 */
GLQ_API glq_status glq_layer_set_prefill_reconstruct(glq_layer layer, int64_t min_batch);

/*
 * glq_dequant_reference -- materialise W^ (fp32, no Hadamards, ws included)
 * into w_dev [m][n] row-major, using the same on-chip decode the GEMV uses.
 * Each value is fp32(ws * fma_f32(rs, cb2, cb1)) (single roundings); from 5
 * bpw one fma_f32 per residual stage in stage order.
 * Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_CUDA.  Asynchronous.
 */
GLQ_API glq_status glq_dequant_reference(glq_layer layer, float *w_dev, void *stream);

/*
 * glq_rht_input / glq_rht_output -- the two Hadamard stages alone, for
 * testing and composition (GLQ v0.3.2 release notes: input_rht,
 * output_rht).  glq_rht_input: xr[B][n] (fp32, device) = H_n (S_in . x).
 * glq_rht_output: y[B][m] (device, y_dtype) = S_out . H_m z, z fp32 device
 * [B][m], with the kernel glq_linear's output stage uses at this batch.
 * Errors as glq_linear.  Asynchronous.
 */
GLQ_API glq_status glq_rht_input(glq_layer layer, const void *x_dev, glq_dtype x_dtype, float *xr_dev,
                         int64_t B, void *stream);
GLQ_API glq_status glq_rht_output(glq_layer layer, const float *z_dev, void *y_dev, glq_dtype y_dtype,
                          int64_t B, void *stream);

/*
 * glq_rht_input_operand -- the input stage of the tensor-core (B > 16)
 * path alone (GLQ v0.3.2 release notes, input_rht), as the fp16 operand
 * the GEMM reads: xh_dev [B][n_pad] fp16 = xr_b 2^e_b, xr = H_n (S_in . x),
 * padding columns zero; row_info_dev [B][4] 32-bit words, word 2 of row b =
 * 2^-e_b as fp32 (the other words unspecified).  The power of two is chosen
 * per row so that the fp16 values stay finite; which one is the kernel's
 * choice.  kernel: 0 the kernel glq_linear runs for this layer; 1 the
 * CUDA-core butterfly kernel (n_pad <= 16384); 2 the tensor-core kernel
 * (512 <= n <= 16384, n a multiple of 256).  Device pointers; x_dev 16-byte
 * aligned.  Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_DTYPE, GLQ_ERR_SHAPE (B >
 * 65535, or a kernel that does not take this row length), GLQ_ERR_CUDA.
 * Asynchronous.
 */
GLQ_API glq_status glq_rht_input_operand(glq_layer layer, const void *x_dev, glq_dtype x_dtype, void *xh_dev,
                                         void *row_info_dev, int64_t B, int kernel, void *stream);

/*
 * glq_layer_selftest_wait -- testing entry point for failure detection: runs
 * one of the bounded device waits the layer's kernels use, on a barrier that
 * only `arrivals` of its two expected arrivals reach (1: it never completes;
 * 2: it completes at once), with the given limit; a wait that runs out
 * reports a timeout through the layer's device error word, as the kernels
 * do, without faulting or hanging the GPU.  kind: 0 the cycle-bounded wait of
 * the tensor-core pipeline (limit in SM clock cycles), 1 its cluster-scope
 * form (same unit), 2 the poll-bounded wait of the codebook-table loads
 * (limit in polls, < 2^32).  Read the outcome with glq_layer_check
 * (GLQ_ERR_TIMEOUT after a timeout, which also clears the word).
 * Errors: GLQ_ERR_INVALID_ARG (kind, arrivals or limit out of range),
 * GLQ_ERR_CUDA.  Asynchronous.
 */
GLQ_API glq_status glq_layer_selftest_wait(glq_layer layer, int kind, int arrivals, int64_t limit, void *stream);

/*
 * glq_gemv_replay -- measurement entry point: re-launches only the codebook
 * GEMV of the most recent glq_linear call on this layer (its activations
 * are read from the device's shared workspace, so no other layer's call may
 * come between; batch B <= min(16, that call's B)),
 * writing the same split-K partial sums.  Lets a caller time the GEMV kernel
 * alone with events on `stream`.  Like glq_linear, it launches the GEMV with
 * programmatic dependent launch, so back-to-back replays overlap one launch's
 * prologue (codebook copy, first index loads) with the previous one's tail,
 * as the product path does.  The decode path's GEMV is the one of
 * "Inference kernels" on the glq 0.5.1 PyPI page (matmul against indices).
 * Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_SHAPE (B out of range or no previous
 * call), GLQ_ERR_CUDA.  Asynchronous.
 */
GLQ_API glq_status glq_gemv_replay(glq_layer layer, int64_t B, void *stream);

/*
 * glq_prefill_replay -- measurement entry point: re-launches only the
 * tensor-core GEMM of the most recent glq_linear call with B > 16 on this
 * layer (its fp16 rotated activations, and its reconstructed W when that
 * call reconstructed one, are read from the device's shared workspace, so
 * no other layer's tensor-core call may come between), for 16 < B <= that
 * call's B, rewriting the same pre-rotation outputs z.  Lets a caller time
 * the GEMM kernel alone with events on `stream`.  The GEMM is the
 * tensor-core path of "Inference kernels" on the glq 0.5.1 PyPI page
 * (matmul against codebook-reconstructed weights).
 * Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_SHAPE (B out of range or no previous
 * call), GLQ_ERR_CUDA.  Asynchronous.
 */
GLQ_API glq_status glq_prefill_replay(glq_layer layer, int64_t B, void *stream);

/*
 * glq_linear_noalloc -- glq_linear for a batch of at most 16 tokens that
 * allocates no device memory, for callers that cannot call cudaMalloc at
 * call time: code running while a CUDA graph is captured, in host
 * callbacks, or under a framework that owns every device allocation.  (The
 * GLQ pages have no counterpart: this is a property of this library's
 * workspace handling.)
 * Instead of the device's shared workspace it uses one fixed device array of
 * GLQ_NOALLOC_SCRATCH_BYTES (8 MiB) that the library defines at file scope;
 * every GPU that loads the library holds it until the process exits.
 * x_dev, y_dev, x_dtype, y_dtype, stream: as glq_linear; 0 <= B <= 16.
 * The first call on a device resolves the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * Calls share the array and it keeps the last call's contents: two calls
 * whose work overlaps on the GPU (other streams, unordered layers) race.
 * A call also writes the layer's own device words (error flag, output-block
 * counters), so calls on one layer must not overlap on the GPU whichever
 * entry point (glq_linear or this one) they use.
 * Results equal glq_linear's, except when glq_linear's split-K partial
 * sums would not fit the array: then the split count is narrowed (possibly
 * to a plan without the fused input transform), and the results agree
 * within the parity bound instead of bitwise.
 * Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_DTYPE, GLQ_ERR_SHAPE (B > 16, or a
 *   layer whose activations plus one split of partial sums exceed the
 *   array), GLQ_ERR_CUDA.  Asynchronous.
 */
#define GLQ_NOALLOC_SCRATCH_BYTES (8u << 20)
GLQ_API glq_status glq_linear_noalloc(glq_layer layer, const void *x_dev, glq_dtype x_dtype,
                                      void *y_dev, glq_dtype y_dtype, int64_t B, void *stream);

/*
 * glq_layer_check -- synchronise `stream`, then read and clear the layer's
 * device error word (set by bounded device-side waits and checks).
 * Returns GLQ_OK, GLQ_ERR_TIMEOUT, GLQ_ERR_DEVICE_CHECK or GLQ_ERR_CUDA.
 */
GLQ_API glq_status glq_layer_check(glq_layer layer, void *stream);

/*
 * glq_decode_plan -- measurement / test entry point: the launch plan a
 * decode call of B tokens (1 <= B <= 16) with 16-byte aligned x and y takes
 * under the layer's current settings: warps per GEMV CTA, row bands, K
 * splits per band, the thread-block cluster size of the split-K reduction
 * (0: global workspace and last-arriving CTA) and whether the input RHT is
 * fused into the GEMV launch (1) or runs as its own kernel (0).  Any output
 * may be NULL.  Errors: GLQ_ERR_INVALID_ARG, GLQ_ERR_SHAPE (B out of range).
 * No counterpart in the pages (a view of this library's scheduling).
 */
GLQ_API glq_status glq_decode_plan(glq_layer layer, int64_t B, int32_t *warps, int32_t *bands,
                                   int32_t *splits, int32_t *cluster, int32_t *fused_input);

/* Layer geometry, for callers sizing buffers.  Any output may be NULL. */
GLQ_API glq_status glq_layer_info(glq_layer layer, int64_t *m, int64_t *n, int32_t *bpw,
                          size_t *device_bytes);

#ifdef __cplusplus
}
#endif

#endif /* GLQ_B200_H */
