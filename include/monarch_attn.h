/*
 * monarch_attn.h -- C ABI of the B200 (sm_100a) Monarch attention forward.
 *
 * The operator (MonarchRT: Efficient Attention for Real-Time Video
 * Generation; gist.science/nl/paper/2602.12271, section "Methodologie": the
 * attention matrix is a product of permutation and block-diagonal matrices;
 * gist.science/zh/paper/2602.12271, section 2.2: blocks aligned with the
 * frame/height/width axes, and tiled Monarch):
 *
 *     out = M V,   M = P^T B2 P B1,
 *
 * per (batch, head) over the N = T*H*W tokens of a video latent, token index
 * n = (t*H + h)*W + w.  B1 is block diagonal over stage-1 blocks (one frame of
 * H*W tokens, or one tile_h x tile_w spatial tile of one frame); P swaps the
 * block index and the in-block index; B2 is block diagonal over the groups of
 * T tokens sharing a spatial position (h, w).  Every diagonal block is a dense
 * softmax attention with scale 1/sqrt(d): stage 1 attends Q to K with values
 * V inside its block, stage 2 attends the same Q and K rows inside a group
 * with the stage-1 outputs as values.
 *
 * Every entry point is plain C: raw pointers, ints, and a cudaStream_t passed
 * as void*.
 *
 * Device memory the library holds itself.  The bf16 / fp16 path needs one
 * 32-bit completion counter per batch-head for each call in flight; the
 * (f*h, w) split also needs a stage-1 scratch of N*d elements per batch-head.
 * Both come from per-device pools that the first call needing them allocates
 * with cudaMalloc and that stay allocated while the library is loaded (never
 * freed, so a pointer captured into a CUDA graph stays valid):
 *   - counters: 64 slots of max(4160, B*heads + 1) words (about 1 MB for up
 *     to 4096 batch-heads): one word per batch-head and the counter from
 *     which the persistent kernel's CTAs claim units.  A larger call allocates a pool of twice the slot size and
 *     retires the old one, so the total stays below twice the largest pool.
 *     A stream keeps its slot while it is among the 64 most recently used;
 *     a stream taking over a slot is ordered after the slot's previous user
 *     with cudaStreamWaitEvent (no host synchronisation).  A stream under
 *     capture pins its slot to itself.
 *   - (f*h, w) scratch: one buffer per device, grown by doubling (outgrown
 *     buffers retired the same way); calls on different streams are ordered
 *     through its event, so such calls on two streams run one after the other.
 * No call frees device memory or synchronises the host (outside
 * MONARCH_ATTN_DEBUG=1).  Encoded TMA tensor maps are cached host-side (1024
 * most recently used, keyed by address, shape, strides, box and type).
 */
#ifndef MONARCH_ATTN_H
#define MONARCH_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
    MONARCH_OK = 0,
    MONARCH_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment, aliasing or enum; nothing launched */
    MONARCH_ERR_UNSUPPORTED = 2, /* valid but outside the library's limits (see below); nothing launched */
    MONARCH_ERR_LAUNCH = 3,      /* a kernel launch failed (cudaGetLastError after launch) */
    MONARCH_ERR_TIMEOUT = 4,     /* a device-side wait gave up (reported by monarch_attn_device_status) */
    MONARCH_ERR_CUDA = 5         /* a CUDA runtime/driver call other than a launch failed */
} monarch_status_t;

/* Element type of q, k, v and out. */
typedef enum {
    MONARCH_DTYPE_F32 = 0,  /* fp32 in and out; exact path on CUDA cores, fp32 accumulation */
    MONARCH_DTYPE_BF16 = 1, /* bf16 in and out; tcgen05 tensor cores, fp32 accumulation and softmax */
    MONARCH_DTYPE_F16 = 2   /* fp16 in and out; as bf16 (P and Y1 held in fp16) */
} monarch_dtype_t;

/* Choice of stage-1 blocks (block alignment: every video axis lies inside one
 * block dimension). */
typedef enum {
    MONARCH_FACT_FRAME = 0, /* block = one frame, m = H*W tokens, b = T blocks */
    MONARCH_FACT_TILED = 1, /* block = one tile_h x tile_w spatial tile of one frame */
    MONARCH_FACT_ROW = 2    /* the (f*h, w) split: block = one frame row (W tokens),
                               group = one column (the T*H tokens sharing w) */
} monarch_fact_t;

/*
 * monarch_attn_fwd -- out = P^T B2 P B1 V (see the top of this file).
 *
 * Arguments
 *   q, k, v   device pointers, inputs, layout [B][heads][N][d] contiguous
 *             (N = T*H*W, token order n = (t*H + h)*W + w), element type
 *             `dtype`.  Read only.
 *   out       device pointer, output, same layout and type.  Must not overlap
 *             q, k or v.  The stage-1 result is kept in `out` between the two
 *             stages (stage 2 reads and overwrites it group by group); out's
 *             prior contents are ignored.
 *   B, heads  batch size and head count, >= 1.
 *   T, H, W   frames, height and width of the token grid, >= 1.
 *   d         head width: 64 or 128.
 *   factorisation  MONARCH_FACT_FRAME, MONARCH_FACT_TILED or MONARCH_FACT_ROW.
 *   tile_h, tile_w tile size for MONARCH_FACT_TILED; must divide H and W
 *             respectively.  Ignored otherwise.
 *
 * MONARCH_FACT_ROW is the (f*h, w) block alignment (gist.science/pt/paper/
 * 2602.12271, "Alinhamento de Blocos"; gist.science/zh/paper/2602.12271,
 * section 2.2): the tokens form a (T*H) x W grid, stage-1 blocks are its rows
 * and stage-2 groups its columns.  It runs as two stage-1 passes of the
 * forward's kernels and keeps the stage-1 result in the device's scratch
 * pool (see the top of this file), so `out` is written only by the second
 * pass.
 *   dtype     MONARCH_DTYPE_BF16, MONARCH_DTYPE_F16 or MONARCH_DTYPE_F32.
 *   stream    cudaStream_t (NULL = legacy default stream) the work is queued on.
 *
 * Limits of this library version (MONARCH_ERR_UNSUPPORTED otherwise): T <= 128
 * (except MONARCH_FACT_ROW); tile_w <= 128 for MONARCH_FACT_TILED; N <= 2^31; a device of compute
 * capability 10.0 (B200).  Pointers must be 16-byte aligned
 * (MONARCH_ERR_INVALID_ARG otherwise).
 *
 * Errors and ownership
 *   The caller owns all four buffers.  Argument errors are reported before
 *   anything is queued.  The call is asynchronous: it returns after queueing
 *   the kernels on `stream`; device faults surface at the caller's next
 *   synchronisation, following CUDA convention.  The bf16 / fp16 kernel is a
 *   cooperative launch (its stage-2 work waits for stage-1 results of other
 *   CTAs): if the device cannot make the whole grid resident at once (for
 *   example under an MPS SM limit) the launch fails and the call returns
 *   MONARCH_ERR_LAUNCH.  Device-side waits are
 *   bounded: a wait that gives up records MONARCH_ERR_TIMEOUT in a device
 *   status word that monarch_attn_device_status() returns.  With the
 *   environment variable MONARCH_ATTN_DEBUG=1 the call synchronises `stream`
 *   and returns that status directly.
 */
int monarch_attn_fwd(const void *q, const void *k, const void *v, void *out,
                     int B, int heads, int T, int H, int W, int d,
                     int factorisation, int tile_h, int tile_w, int dtype,
                     void *stream);

/*
 * monarch_attn_fwd_strided -- monarch_attn_fwd for q, k, v and out laid out
 * with the given element strides: element c of token n of (batch b, head h)
 * is at b*stride_b + h*stride_h + n*stride_n + c in each of the four tensors
 * (the d features of a token are contiguous).  [B][heads][N][d] is
 * (heads*N*d, N*d, d); [B][N][heads][d], the layout of many video DiT
 * codebases, is (N*heads*d, d, heads*d).  Token order within N stays
 * n = (t*H + h)*W + w.
 *
 * Errors, besides monarch_attn_fwd's: MONARCH_ERR_INVALID_ARG if a stride is
 * below 1, if token rows of one tensor would overlap (sorted by stride, each
 * stride must be at least the next smaller stride times its extent, and the
 * smallest at least d), or, for 16-bit dtypes, if a stride is not a multiple
 * of 8 elements (16 bytes); MONARCH_ERR_UNSUPPORTED for MONARCH_FACT_TILED
 * and MONARCH_FACT_ROW with strides other than the contiguous ones.
 */
int monarch_attn_fwd_strided(const void *q, const void *k, const void *v, void *out,
                             int B, int heads, int T, int H, int W, int d,
                             int factorisation, int tile_h, int tile_w, int dtype,
                             long long stride_b, long long stride_h, long long stride_n,
                             void *stream);

/*
 * monarch_attn_fwd_host -- the same operator for inputs and output in host
 * memory.  Queues on `stream`: copies of h_q, h_k, h_v into the caller's
 * device buffers d_q, d_k, d_v (one cudaMemcpyAsync each), monarch_attn_fwd
 * on the device buffers, and a copy of d_out back into h_out; then waits for
 * the stream.  Host buffers should be pinned for asynchronous copies.  All
 * eight buffers are owned by the caller and hold B*heads*N*d elements of
 * `dtype`; the device buffers follow monarch_attn_fwd's rules.
 * Returns after h_out is written, or with the first error.
 */
int monarch_attn_fwd_host(const void *h_q, const void *h_k, const void *h_v, void *h_out,
                          void *d_q, void *d_k, void *d_v, void *d_out,
                          int B, int heads, int T, int H, int W, int d,
                          int factorisation, int tile_h, int tile_w, int dtype,
                          void *stream);

/*
 * monarch_attn_fwd_host_pipelined -- monarch_attn_fwd_host with the copies
 * overlapped with the computation.  The B*heads (batch, head) problems are
 * independent; the call splits them into `nchunks` chunks of consecutive
 * batch-heads and pipelines them: chunk c+1 is uploaded while chunk c is
 * computed (on `stream`, one monarch_attn_fwd call per chunk) and chunk c-1
 * is downloaded.  Uploads and downloads run on two streams the library
 * creates on first use, one pair per device, and keeps (calls from several
 * threads on one device share them); the first upload waits for work
 * already queued on `stream`.
 * Results equal monarch_attn_fwd_host's bit for bit (each problem's
 * arithmetic does not depend on the chunking).  Host buffers must be pinned
 * for the copies to overlap.  nchunks >= 1 (capped at B*heads).  Arguments,
 * buffer rules and status codes as monarch_attn_fwd_host; returns after h_out
 * is written, or with the first error.
 */
int monarch_attn_fwd_host_pipelined(const void *h_q, const void *h_k, const void *h_v, void *h_out,
                                    void *d_q, void *d_k, void *d_v, void *d_out,
                                    int B, int heads, int T, int H, int W, int d,
                                    int factorisation, int tile_h, int tile_w, int dtype,
                                    int nchunks, void *stream);

/*
 * monarch_attn_fwd_profiled -- monarch_attn_fwd that also records CUDA events
 * on `stream` so a caller can time each kernel launch of the call:
 * events[0] before the first launch and events[i + 1] after launch i.
 * `events` holds `nevents` cudaEvent_t handles created by the caller
 * (entries beyond what the call needs are left untouched; NULL entries are
 * skipped).  *nlaunch (if not NULL) receives the number of kernel launches
 * the call queued: 1 for bf16 and fp16 (both stages in one persistent
 * kernel), 2 for fp32 (stage 1, then stage 2), and 2 for MONARCH_FACT_ROW in
 * every dtype (the rows pass, then the columns pass).  Same arguments, rules and status codes as
 * monarch_attn_fwd otherwise.
 */
int monarch_attn_fwd_profiled(const void *q, const void *k, const void *v, void *out,
                              int B, int heads, int T, int H, int W, int d,
                              int factorisation, int tile_h, int tile_w, int dtype,
                              void *stream, void **events, int nevents, int *nlaunch);

/* Largest B*heads monarch_attn_fwd_noalloc accepts (size of its static
 * counter array: one 32-bit word per batch-head plus the unit-claim counter,
 * about 16 KB per device). */
#define MONARCH_NOALLOC_MAX_BH 4096

/*
 * monarch_attn_fwd_noalloc -- monarch_attn_fwd for bf16 that allocates no
 * device memory.  No counterpart in the pages: it exists for callers that
 * cannot allocate once running (a real-time generation loop, where
 * monarch_attn_fwd's first call on a device, or its first call with more
 * batch-heads than any before, would cudaMalloc its counter pool, which can
 * stall behind other work on the device; or a host whose device memory is
 * all held by its own pool).
 *
 * Arguments, layout, ownership and status codes are those of
 * monarch_attn_fwd with dtype = MONARCH_DTYPE_BF16.  Scratch: the per-batch-
 * head completion counters live in one static device array per device of
 * MONARCH_NOALLOC_MAX_BH words; B*heads above that returns
 * MONARCH_ERR_UNSUPPORTED before anything is queued, and so does
 * MONARCH_FACT_ROW (its stage-1 result needs the library's scratch buffer).  Those counters must be
 * zero when the kernel starts; every call zeroes them with a cudaMemsetAsync
 * on `stream` ahead of its launch.  The first call on each device does a
 * one-time set-up on the host (the array's address, the kernel's shared-
 * memory attribute, the tensor-map encoder); make that first call before
 * beginning any stream capture.
 *
 * Calls race when they overlap: every call on a device uses the same
 * counters, so two calls whose work can run at the same time (on different
 * streams, or from different host threads without ordering) may let stage 2
 * read unfinished stage-1 results, or time out.  Queue such calls on one
 * stream, or order them with events.
 */
int monarch_attn_fwd_noalloc(const void *q, const void *k, const void *v, void *out,
                             int B, int heads, int T, int H, int W, int d,
                             int factorisation, int tile_h, int tile_w, void *stream);

/*
 * monarch_attn_fwd_chunk -- one chunk of autoregressive generation: the
 * forward of T_new new frames with the T_old frames before them as context.
 * The pages' main model generates video autoregressively (gist.science/it/
 * paper/2602.12271, problem statement) and their kernels split the query
 * frames into chunks (gist.science/zh/paper/2602.12271, section 2.2); they
 * define no cache.  Reading used here: stage 1 (frame or tiled blocks) never
 * crosses frames, so it runs on the new frames alone; stage 2 of a new query
 * at spatial position pos attends over the keys of all T_old + T_new frames
 * at pos, with their stage-1 outputs as values.  So the context is the keys
 * and stage-1 outputs of the earlier frames.  For the last chunk of a clip,
 * with the context taken from a forward of the whole clip, `out` equals that
 * forward's rows for those frames.
 *
 * q, k, v: the new frames, [B][heads][T_new*H*W][d] contiguous (as
 * monarch_attn_fwd with T = T_new).  k_cache, y1_cache: keys and stage-1
 * outputs of the context, [B][heads][T_old*H*W][d] contiguous, same dtype;
 * ignored (may be NULL) when T_old = 0.  out: the chunk's output; y1_new:
 * the stage-1 output of the new frames (to append to y1_cache for the next
 * chunk, with k appended to k_cache); both [B][heads][T_new*H*W][d],
 * written, previous contents ignored.  No output may overlap an input or the
 * other output.  All pointers 16-byte aligned.  dtype, d, factorisation and
 * tiles as monarch_attn_fwd (MONARCH_FACT_FRAME or _TILED); 1 <= T_new <=
 * 128, T_old >= 0.  Two launches on `stream`: the forward's stage-1 kernel
 * (tcgen05 tensor cores for bf16/fp16, CUDA cores for fp32), then stage 2,
 * one warp per (batch-head, position) (warp-level mma.sync tensor-core tiles
 * for bf16/fp16, CUDA cores for fp32).  Y1 is held in the input dtype.  Status codes as monarch_attn_fwd;
 * MONARCH_ERR_INVALID_ARG also for T_old < 0 or missing context pointers.
 */
int monarch_attn_fwd_chunk(const void *q, const void *k, const void *v,
                           const void *k_cache, const void *y1_cache, void *out, void *y1_new,
                           int B, int heads, int T_old, int T_new, int H, int W, int d,
                           int factorisation, int tile_h, int tile_w, int dtype, void *stream);

/*
 * monarch_attn_fwd_chunk_profiled -- monarch_attn_fwd_chunk recording CUDA
 * events around its launches as monarch_attn_fwd_profiled does: events[0]
 * before the first launch, events[i + 1] after launch i; *nlaunch receives 2
 * (stage 1, then stage 2).  Same arguments, rules and status codes as
 * monarch_attn_fwd_chunk otherwise.
 */
int monarch_attn_fwd_chunk_profiled(const void *q, const void *k, const void *v,
                                    const void *k_cache, const void *y1_cache, void *out,
                                    void *y1_new, int B, int heads, int T_old, int T_new, int H,
                                    int W, int d, int factorisation, int tile_h, int tile_w,
                                    int dtype, void *stream, void **events, int nevents,
                                    int *nlaunch);

/*
 * monarch_attn_bwd -- gradients of out = P^T B2 P B1 V (as monarch_attn_fwd)
 * with respect to q, k and v for an upstream gradient dout.  The pages state
 * that their kernels run the backward pass too (gist.science/nl/paper/
 * 2602.12271, "Methodologie"; gist.science/zh/paper/2602.12271, section 2.2);
 * the gradient itself follows from the forward by the chain rule.
 *
 * Each stage's backward is the attention backward of its diagonal blocks:
 * with P = softmax(Q K^T / sqrt(d)), upstream dY, values Vals and output Y,
 * dVals = P^T dY, dS = P * (dY Vals^T - rowsum(dY * Y)), dQ = dS K / sqrt(d),
 * dK = dS^T Q / sqrt(d).  Stage 2 (values Y1, upstream dout) yields dY1;
 * stage 1 (values V, upstream dY1) yields dV; dQ and dK sum both stages.
 *
 * Layout [B][heads][N][d] contiguous, as monarch_attn_fwd.  q, k, v, dout are
 * read; dq, dk, dv are written (previous contents ignored), all of type
 * `dtype`.  workspace: caller-owned device memory of at least
 * monarch_attn_bwd_workspace_size(...) bytes; its contents on entry do not
 * matter.  No output or the workspace may overlap an input or another output.
 * Returns MONARCH_ERR_INVALID_ARG for bad pointers, sizes, alignment (16
 * bytes), overlap or a too-small workspace.  Asynchronous on `stream`.
 *
 * dtype MONARCH_DTYPE_BF16 / MONARCH_DTYPE_F16 (tensor cores; every
 * factorisation, including MONARCH_FACT_ROW): the workspace holds the
 * recomputed Y1 and O and dY1 (16-bit), per-row rowsum terms and each
 * stage's per-row LSE (fp32) and stage 2's dQ and dK parts (fp32):
 * N*(6d + 12 + 8d) bytes per batch-head.  The forward's kernel recomputes Y1
 * and O, leaving each stage's row LSE as it goes; then per stage the CTAs of
 * a query-outer kernel (dQ) and of a key-outer kernel (dK and dValues) run,
 * in one launch, on tcgen05 with fp32 accumulation and 16-bit P, dS and dY1;
 * stage 1's kernels
 * add stage 2's parts and write dq, dk, dv.  Every gradient row has one
 * owning CTA, so the result is deterministic.  Limits as monarch_attn_fwd.
 *
 * dtype MONARCH_DTYPE_F32 (CUDA cores, frame and tiled factorisations): the
 * workspace holds the recomputed stage-1 output and its gradient (2*N*d
 * floats per batch-head).  Limits: T <= 128, and for the stage-1 blocks 8*m
 * floats of shared memory (m <= 6400 tokens per block).  dk and dv are
 * accumulated with atomic adds, so repeated calls can differ in the last
 * bits.
 */
int monarch_attn_bwd(const void *q, const void *k, const void *v, const void *dout,
                     void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                     int B, int heads, int T, int H, int W, int d,
                     int factorisation, int tile_h, int tile_w, int dtype, void *stream);

/* Workspace bytes monarch_attn_bwd needs for these sizes (0 if unsupported). */
size_t monarch_attn_bwd_workspace_size(int B, int heads, int T, int H, int W, int d, int dtype);

/*
 * monarch_attn_bwd_profiled -- monarch_attn_bwd that also records CUDA events
 * (cudaEvent_t passed as void*, created by the caller) on `stream`:
 * events[0] before the first launch and events[i] after the i-th phase.
 * Phases, 16-bit dtypes: 1 Y1 recomputation, 2 O recomputation, 3 stage-2
 * backward (row sums, then the dQ and dK/dV CTAs in one launch), 4 stage-1
 * backward (the same, writing dq, dk, dv); fp32: 1 the whole backward.  *nlaunch receives
 * the number of phases recorded.  Events beyond `nevents` are not recorded.
 */
int monarch_attn_bwd_profiled(const void *q, const void *k, const void *v, const void *dout,
                              void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                              int B, int heads, int T, int H, int W, int d,
                              int factorisation, int tile_h, int tile_w, int dtype, void *stream,
                              void **events, int nevents, int *nlaunch);

/* Human-readable text of a status code; never NULL, owned by the library. */
const char *monarch_attn_strerror(int status);

/*
 * monarch_attn_device_status -- synchronises `stream`, then returns
 * MONARCH_ERR_TIMEOUT if any kernel of this library on the current device
 * recorded a timed-out wait since the last reset, MONARCH_ERR_CUDA if the
 * synchronisation itself failed, else MONARCH_OK.  With reset != 0 the
 * device status word is cleared afterwards.
 */
int monarch_attn_device_status(void *stream, int reset);

/*
 * monarch_attn_selftest_timeout -- exercises the bounded-wait machinery:
 * launches one block whose thread waits on a barrier that nothing completes,
 * for at most `limit_cycles` SM clock cycles, then records a timeout in the
 * device status word and returns.  Returns the value monarch_attn_device_status
 * would (MONARCH_ERR_TIMEOUT when the machinery works) and clears the word.
 * No counterpart in the pages: this is error-path test support.
 */
int monarch_attn_selftest_timeout(long long limit_cycles, void *stream);

/* Version of this library as MAJOR*10000 + MINOR*100 + PATCH. */
int monarch_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MONARCH_ATTN_H */
