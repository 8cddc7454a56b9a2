/*
 * rotate_attn.h -- C ABI of the RotateAttention INT4 attention forward for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "RotateAttention: RoPE-Aware Rotation and Range Rectification for
 * INT4 Quantized Attention in Video Generation" (arXiv 2607.02584), as
 * described on its review page (pith summary, core claim, "What carries the
 * argument", free-parameter ledger, abstract, Fig. 2 and Fig. 3 captions).
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers, 16-byte aligned, row-major and contiguous.
 *     fp16 tensors are [B][H][N][d] with d = 128.  (ra_int4_attention_host
 *     alone takes host q, k, v, o.)
 *   - The caller owns all memory.  The library allocates and frees nothing on
 *     any call; it only reads and writes the buffers it is given.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns without synchronising, except ra_check_device_error
 *     and ra_int4_attention_host.
 *   - Errors are status codes; nothing throws or aborts across the ABI.
 *     Argument errors are found on the host before any launch and nothing is
 *     enqueued then.  ra_last_error_detail() gives a one-line reason for the
 *     last non-OK status of the calling thread.
 *   - Device-side faults are not raised as CUDA errors: every bounded wait
 *     and every self-check in the kernels records a code in the workspace's
 *     error word; ra_check_device_error() reads and clears it.
 *   - Calls that share a workspace must not overlap on the GPU.
 */
#ifndef ROTATE_ATTN_H
#define ROTATE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RA_OK = 0,
    RA_ERR_INVALID_ARG = 1,     /* bad shape, split, mode, null or misaligned pointer */
    RA_ERR_UNSUPPORTED = 2,     /* valid in principle, not built (e.g. d != 128) */
    RA_ERR_WORKSPACE = 3,       /* workspace too small or not prepared for this problem */
    RA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
    RA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out */
    RA_ERR_DEVICE_BOUNDS = 6    /* a device-side self-check found a bad index */
} ra_status;

typedef enum {
    RA_ROT_NONE = 0,            /* RoPE only */
    RA_ROT_INTERLEAVED = 1,     /* H2 on adjacent dims, merged into RoPE (Fig. 3) */
    RA_ROT_HALF = 2,            /* H2 on (i, i + d_s/2) in each segment (Fig. 3) */
    RA_ROT_FULL = 3,            /* dense rotation over all of head_dim after RoPE: the
                                 * normalised 128-point Walsh-Hadamard transform (the
                                 * "Full" rotation the pages compare against, Figs. 4-5;
                                 * the matrix is not given there).  Computed as the fast
                                 * transform in fp32, strides 1, 2, ..., 64, then one
                                 * multiply by fp32(1/sqrt(128)). */
    RA_ROT_BLOCKS_INTERLEAVED = 4, /* caller's 2x2 orthogonal block per adjacent pair
                                 * (learned rotations, Sec. 4.1 / Fig. 6), merged into
                                 * RoPE per (position, pair) like the Interleaved H2 */
    RA_ROT_BLOCKS_HALF = 5      /* caller's 2x2 orthogonal block per (i, i + d_s/2)
                                 * pair, applied after RoPE like the Half H2 */
} ra_rot_mode;

/* Quantisation of P = exp(s - m) in [0, 1] for the P.V product.
 * RA_P_RANGE_OPTIMIZED (the method): code = rne(15 P) - 8 in [-8, 7], the
 *   full signed INT4 range, with the zero-point corrected through the V
 *   column sums ("What carries the argument"; free-parameter ledger, Sec. 4.2).
 * RA_P_SYMMETRIC: plain symmetric INT4, code = rne(7 P) in [0, 7], no
 *   zero-point (the baseline that leaves half the codes unused, abstract); the
 *   pages' referee report and the "If this is right" list suggest disabling
 *   the range-optimised map for low-entropy (image-to-video) attention. */
typedef enum {
    RA_P_RANGE_OPTIMIZED = 0,
    RA_P_SYMMETRIC = 1
} ra_p_mode;

/* One attention problem.  Tokens: N = F*Hh*W video tokens in frame-major
 * order (frame slowest, column fastest) followed by n_text text tokens, which
 * get no RoPE but do get the rotation.  head_dim d is split into three RoPE
 * segments split[0..2] (frame, height, width; each even, sum = d); pair j of
 * segment s (dims o_s+2j, o_s+2j+1) turns by pos_s * theta^(-2j/split[s]). */
typedef struct {
    int B, H, d;
    int F, Hh, W, n_text;
    int split[3];
    double theta;               /* RoPE base, e.g. 10000.0 */
    int rot;                    /* ra_rot_mode */
    int p_mode;                 /* ra_p_mode (INT4 attention only; 0 = the method) */
    int v_rot;                  /* 1: the INT4 path multiplies every V row by the
                                 * normalised 128-point Walsh-Hadamard matrix before
                                 * quantising it and every output row by its transpose
                                 * (a stand-in for the Hadamard the pages fuse into V
                                 * offline: review page summary); 0: V as given */
    const double *blocks;       /* host, d/2 x 4: block p = {r00, r01, r10, r11}, row
                                 * major, rows orthonormal to 1e-6; needed for the
                                 * BLOCKS modes (NULL otherwise).  Pair p of segment s
                                 * is p = o_s / 2 + j (dims o_s + 2j, o_s + 2j + 1 for
                                 * INTERLEAVED; o_s + j, o_s + j + d_s/2 for HALF);
                                 * (z_a, z_b) = R (y_a, y_b). */
} ra_problem;

/* Quantised Q, K, V as produced by ra_rotate_quantize_qkv (device memory).
 * N_pad = N rounded up to a multiple of 128; padded tokens hold code 0.
 *   q4, k4 : uint8 [B][H][N_pad][64]  two INT4 codes per byte, channel 2c in
 *            the low nibble and 2c+1 in the high nibble, two's complement,
 *            codes in [-7, 7]
 *   v4t    : uint8 [B][H][N_pad/128][128][64]  V transposed per 128-token
 *            tile: tile t, channel c, byte b holds tokens 128t+2b (low
 *            nibble) and 128t+2b+1 (high nibble); each tile is one contiguous
 *            8 KB block
 *   sq, sk : float [B][H][N_pad/64]   one scale per 64-token block (amax/7)
 *   sv     : float [B][H][128]        one scale per channel over all N tokens
 *   vsum   : int32 [B][H][N_pad/64][128]  per-64-token-block column sums of
 *            the V codes (the zero-point correction term of P.V) */
typedef struct {
    uint8_t *q4, *k4, *v4t;
    float *sq, *sk, *sv;
    int32_t *vsum;
} ra_qkv4;

typedef void *ra_stream;        /* cudaStream_t */

/* Sequence length N and padded length N_pad of a problem (-1 if invalid). */
int ra_seq_len(const ra_problem *p);
int ra_seq_pad(const ra_problem *p);

/* Checks a problem: B, H >= 1; d == 128 (else RA_ERR_UNSUPPORTED); grid
 * sizes >= 0 with N >= 1; split entries even, positive, summing to d;
 * rot in ra_rot_mode; theta > 0; B*H <= 65535; N <= RA_MAX_TOKENS (else
 * RA_ERR_UNSUPPORTED).  The INT4 attention accumulates P.V in int32 in
 * tensor memory, on top of a fixed offset of 0x4B400000 (1,262,485,504): with
 * V codes widened to 16 * code (|.| <= 112) and P weights code + 8 <= 15 per
 * key, a row's sum stays within 112 * 15 * N of the offset, which
 * RA_MAX_TOKENS keeps inside the int32 range. */
#define RA_MAX_TOKENS (1 << 19)
ra_status ra_validate(const ra_problem *p);

/* Bytes of one device buffer that holds all of ra_qkv4 (sub-buffers aligned
 * to 256 bytes), and the binding of such a buffer into an ra_qkv4. */
size_t ra_qkv4_bytes(const ra_problem *p);
ra_status ra_qkv4_bind(const ra_problem *p, void *base, size_t bytes, ra_qkv4 *out);

/* Workspace: error word, RoPE/rotation tables, V channel-amax scratch (all
 * the prologue needs); the INT4 attention's INT8 operand images of Q, K and
 * V^T, which ra_int4_attention_fwd expands from the packed codes on every
 * call (3 * B*H*N_pad*128 bytes); and, when with_fp16_path != 0, the FP16
 * path's position-encoded Q, K and transposed V (3 * B*H*N_pad*128 fp16).
 * Device memory owned by the caller. */
size_t ra_workspace_bytes(const ra_problem *p, int with_fp16_path);

/* Builds the RoPE/rotation coefficient tables on the host (float64 libm,
 * each coefficient rounded once to fp32), copies them into the workspace
 * with cudaMemcpyAsync on `stream`, clears the error word and records the
 * problem's signature.  Call once per (problem, workspace) before the other
 * calls; they check the signature on the device and report
 * RA_ERR_WORKSPACE through ra_check_device_error when it does not match.
 * The signature covers what the tables depend on (d, grid, text tokens,
 * split, theta, rotation, pair blocks), not B or H: a workspace prepared
 * once serves problems that differ only in batch or head count, as long as
 * it is large enough for them. */
ra_status ra_prepare(const ra_problem *p, void *workspace, size_t workspace_bytes, ra_stream stream);

/* Fused prologue: 3D RoPE and the RoPE-aware rotation of Q and K, per
 * 64-token-block symmetric INT4 quantisation of Q and K, per-channel
 * symmetric INT4 quantisation of V with transposed packing and column sums.
 * q, k, v: fp16 [B][H][N][128]; out: bound by ra_qkv4_bind.
 * ("What carries the argument"; Fig. 3 caption; free-parameter ledger.) */
ra_status ra_rotate_quantize_qkv(const ra_problem *p, const void *q, const void *k, const void *v,
                                 const ra_qkv4 *out, void *workspace, size_t workspace_bytes,
                                 ra_stream stream);

/* INT4 attention forward: S = Q K^T on INT8 tensor cores (the INT4 codes
 * are first expanded to INT8 operand images in the workspace, two launches
 * per call), online softmax over 128-key tiles, P = exp(s - m) quantised to
 * rne(15 P) - 8, P.V with the zero-point correction, fp16 output.
 * in: from ra_rotate_quantize_qkv; o: fp16 [B][H][N][128].
 * Workspace: ra_workspace_bytes(p, 0) bytes at least.
 * (Abstract; Sec. 4.2 as summarised in the referee report and ledger.) */
ra_status ra_int4_attention_fwd(const ra_problem *p, const ra_qkv4 *in, void *o,
                                void *workspace, size_t workspace_bytes, ra_stream stream);

/* FP16 path (the pages' mixed-precision fallback, abstract and Sec. 5.1):
 * 3D RoPE in fp32 rounded to fp16 (no rotation: an orthogonal rotation does
 * not change full-precision attention), then FlashAttention with fp32
 * accumulation.  q, k, v, o: fp16 [B][H][N][128].  Needs a workspace sized
 * with with_fp16_path != 0. */
ra_status ra_fp16_attention_fwd(const ra_problem *p, const void *q, const void *k, const void *v,
                                void *o, void *workspace, size_t workspace_bytes, ra_stream stream);

/* ---- INT4 forward on host buffers ------------------------------------- */

/* Device bytes of the staging buffer ra_int4_attention_host needs (0 if the
 * problem or heads_per_chunk is invalid). */
size_t ra_host_staging_bytes(const ra_problem *p, int heads_per_chunk);

/* The whole INT4 path (ra_rotate_quantize_qkv, then ra_int4_attention_fwd)
 * from HOST q, k, v to HOST o, all fp16 [B][H][N][128], with the transfers
 * overlapped with the kernels.  The B*H heads, flattened, are processed in
 * chunks of consecutive heads, each chunk as a problem of its own with B = 1
 * (every step of the path is independent per head, so the results are
 * bit-identical to the device-buffer calls).  heads_per_chunk > 0: chunks of
 * that many heads; 0: chunks of about B*H/8 heads, entered by the ramp 1, 1,
 * 2, 2, 3, 3, 4, 4, ... and left by ..., 3, 2, 1 heads (ra_host_chunks lists
 * them), so that the kernels start after a one-head copy and the last copy
 * back is of one head.  Three staging slots let the inputs of up to two
 * chunks ahead be copied in while chunk c is computed, and the output of
 * chunk c-1 is copied out meanwhile; chunks alternate between `stream` and a
 * second compute stream so that the kernels of chunk c+1 start on the SMs
 * chunk c's last wave leaves idle.  The call creates and destroys its three
 * extra streams and eleven events.  The
 * copies overlap only if the host buffers are page-locked (cudaHostAlloc /
 * cudaHostRegister); pageable buffers give the same result without the
 * overlap.
 * staging: device memory owned by the caller, 256-byte aligned, at least
 * ra_host_staging_bytes(p, heads_per_chunk) bytes: three slots, each with q,
 * k, v, o, the quantised tensors and a workspace for the largest chunk.  The
 * call blocks until o is written and the device error words are checked,
 * so it returns any status ra_check_device_error can.  The staging buffer
 * must not be used by other work while the call runs. */
ra_status ra_int4_attention_host(const ra_problem *p, const void *q, const void *k, const void *v, void *o,
                                 int heads_per_chunk, void *staging, size_t staging_bytes, ra_stream stream);

/* Synchronises `stream`, reads and clears the workspace's error word.
 * Returns RA_OK, RA_ERR_DEVICE_TIMEOUT, RA_ERR_DEVICE_BOUNDS or
 * RA_ERR_WORKSPACE (signature mismatch), or RA_ERR_CUDA. */
ra_status ra_check_device_error(void *workspace, ra_stream stream);

const char *ra_status_string(ra_status s);
const char *ra_last_error_detail(void);

/* ---- allocation-free prologue ------------------------------------------ */

/* Size of the fixed device scratch behind ra_rotate_quantize_qkv_noalloc. */
#define RA_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/* The same fused prologue as ra_rotate_quantize_qkv (same kernels, same
 * bit-exact outputs), for callers that cannot give the library any device
 * memory beyond their own inputs and outputs: for example an engine plugin
 * whose enqueue hook must not allocate (cudaMalloc may synchronise the device
 * or fail mid-run), or a program whose device memory is fully laid out in
 * advance.  The paper has no counterpart; this is a deployment variant.
 *
 * Its scratch -- error word, RoPE/rotation tables and the per-channel V amax
 * -- lives in one fixed array of RA_NOALLOC_SCRATCH_BYTES inside this
 * library, which every GPU that loads the library holds until the process
 * exits.  Problems whose scratch would not fit (about 512 bytes per head plus
 * 16 bytes per RoPE table slot -- 4 ceil(split[s] / 8) slots per position of
 * segment s -- plus 16 bytes per channel pair and a 256-byte header) are
 * rejected with
 * RA_ERR_WORKSPACE before anything is enqueued.  The call allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine); it copies the
 * tables from static host memory with cudaMemcpyAsync on `stream` (a pageable
 * copy, so the call returns once the copy is staged, after the work queued
 * before it on `stream`), then launches the prologue.  The first call on each
 * device also looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and keeps it; make that first call before any stream
 * capture.  A call that fails drops the kept address, so it is looked up
 * again after a device reset (cudaDeviceReset invalidates it).  Every call
 * shares the one array and leaves its contents behind; what must start at
 * zero (the error word, the V amax) is cleared by each call.  Calls whose GPU
 * work overlaps (other streams, other host threads) race on the array:
 * serialise them.  ra_noalloc_check_device_error reports what the kernels
 * found, a table signature that does not match its problem (the sign of such
 * a race) included.
 * q, k, v, out: as for ra_rotate_quantize_qkv. */
ra_status ra_rotate_quantize_qkv_noalloc(const ra_problem *p, const void *q, const void *k, const void *v,
                                         const ra_qkv4 *out, ra_stream stream);

/* The allocation-free counterpart of ra_check_device_error: synchronises
 * `stream`, reads and clears the error word of the fixed scratch of the
 * current device.  Returns RA_OK, RA_ERR_WORKSPACE (the tables in the scratch
 * were not the problem's: overlapping calls), RA_ERR_DEVICE_TIMEOUT,
 * RA_ERR_DEVICE_BOUNDS or RA_ERR_CUDA.  Allocates nothing. */
ra_status ra_noalloc_check_device_error(ra_stream stream);

/* ---- test hooks ------------------------------------------------------- */

/* Number of floats of the coefficient table and the table itself, as
 * ra_prepare uploads it: for segment s, position pos in [0, P_s) with
 * P = (F, Hh, W), pair j: {cos, sin, alpha, beta} at
 * 4 * (off_s + pos * 4 q_s + (j % 4) q_s + j / 4), q_s = ceil(split[s] / 8),
 * off_0 = 0, off_{s+1} = off_s + P_s * 4 q_s (the other slots of a block are
 * zero); then the d/2 pair blocks (r00, r01, r10, r11), zero unless the
 * rotation takes caller blocks. */
size_t ra_tables_floats(const ra_problem *p);
ra_status ra_build_tables_host(const ra_problem *p, float *out, size_t n_floats);

/* Runs the INT4 attention for one (b*H + h, 128-row query tile) through the
 * same kernel and records, for KV tile kv_tile, the int32 S tile
 * (s_out: device int32 [128][128], S[row][key], keys past N = 0) and the P
 * codes (p_out: device int8 [128][128], code in [-8, 7], -128 past N). */
ra_status ra_debug_int4_tile(const ra_problem *p, const ra_qkv4 *in, int bh, int q_tile, int kv_tile,
                             int32_t *s_out, int8_t *p_out, void *workspace, size_t workspace_bytes,
                             ra_stream stream);

/* The chunk sizes (heads per chunk, in order) ra_int4_attention_host would
 * use: writes min(count, max_chunks) of them to sizes (may be NULL) and
 * returns the count, or -1 for an invalid problem or heads_per_chunk < 0. */
int ra_host_chunks(const ra_problem *p, int heads_per_chunk, int *sizes, int max_chunks);

/* Sets the wall-clock limit of every bounded device-side wait, in
 * microseconds (0 restores the default of 2 s); a test sets 1 and runs
 * ra_debug_timeout_probe, whose kernel waits on a barrier that nothing arms
 * and must return RA_ERR_DEVICE_TIMEOUT via ra_check_device_error. */
void ra_debug_set_wait_timeout_us(uint32_t microseconds);
ra_status ra_debug_timeout_probe(void *workspace, size_t workspace_bytes, ra_stream stream);

/* y[i] = 2^x[i] as the INT4 attention kernel computes it for the P code
 * (the hardware ex2.approx, flush-to-zero), for n device floats: a test
 * measures its relative error against float64, the bound behind the
 * "ambiguous key" reading of P-code parity. */
ra_status ra_debug_ex2(const float *x, float *y, int n, ra_stream stream);

/* ---- measurement hook --------------------------------------------------- */

/* Enqueues the INT8 tensor-core rate probe behind the roofline of the INT4
 * attention (the pages state no peak; this measures the denominator): `ctas`
 * CTAs of one per SM, each with one thread issuing `iters` x 4 back-to-back
 * tcgen05.mma.kind::i8 M128 x n x K32 (n = 128 or 256) on shared-memory
 * operands laid out as the attention kernel's, so one launch performs
 * ctas * iters * 4 * 2 * 128 * n * 32 integer operations.  The caller times it
 * with CUDA events on `stream`.  workspace: device, >= 256 bytes (its error
 * word records a timed-out completion wait; read it with
 * ra_check_device_error). */
ra_status ra_measure_mma_i8(int n, int iters, int ctas, void *workspace, size_t workspace_bytes,
                            ra_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* ROTATE_ATTN_H */
