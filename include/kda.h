/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library.
 *
 * The operation.  KDA is a gated delta-rule recurrence with one forgetting
 * factor per key channel.  For each (sequence, head), with state S (d_k x d_v):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t          (the query reads the updated state)
 *
 * Source: "Kimi K3" open-weights field notes (ailearn.mscapital.top/kimi-k3.html),
 * panel "KDA 单头递归" (KDA single-head recurrence): alpha_t = exp(g_t) is the
 * per-channel forgetting, beta_t the per-token write strength, the old state is
 * decayed per channel first and then corrected and written by the delta rule.
 * The same page's panel "g ∈ (-5, 0)" bounds the log-decay; the library relies
 * on g <= 0 (see the preconditions below).  No query scaling or normalisation
 * happens inside the library: callers pass q and k as they want them used.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous.  Alignment: prefill q, k, v, h0, hT and the workspace 16
 *     bytes, g 8 bytes (16 on the tensor-core path, bf16 with d = 128), o two
 *     elements; the decode state S 16 bytes; everything else its element size.  A violation returns KDA_ERR_MISALIGNED.  The library never
 *     allocates device memory and never synchronises the stream in the compute
 *     entry points.
 *   - q, k, g are [.., H, d_k]; v, o are [.., H, d_v]; beta is [.., H];
 *     states are [N, H, d_k, d_v] fp32 (d_k rows, d_v columns).
 *   - q, k, v and o share one dtype (kda_dtype); g, beta and states are fp32.
 *   - Arguments are validated on the host before any launch; a rejected call
 *     launches nothing and returns a status.  No C++ exception crosses the ABI.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  Launch failures are reported as KDA_ERR_CUDA.
 *   - Supported head sizes: d_k == d_v in {32, 64, 128}.  bf16 with d = 128 runs
 *     the tensor-core chunkwise path; every other supported combination runs the
 *     fp32 CUDA-core chunkwise path.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, bad dtype     */
    KDA_ERR_UNSUPPORTED_SHAPE = 2,    /* head size not supported                   */
    KDA_ERR_MISALIGNED = 3,           /* a pointer breaks its alignment rule       */
    KDA_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes < kda_fwd_workspace_size(...)    */
    KDA_ERR_CUDA = 5,                 /* a CUDA launch or query failed             */
    KDA_ERR_DEVICE_TIMEOUT = 6,       /* a bounded device-side wait gave up        */
    KDA_ERR_BAD_SEQLENS = 7,          /* cu_seqlens not monotone / out of range    */
    KDA_ERR_EXCEEDS_STATIC_SCRATCH = 8, /* kda_fwd_noalloc: problem too large      */
    KDA_ERR_CHECKPOINT_CAPACITY = 9,  /* kda_fwd_checkpointed: more checkpoints than slots */
    KDA_ERR_DEBUG_BOUNDS = 10,        /* debug build: a device-side bounds check failed */
    KDA_ERR_BAD_ACCEPTED = 11         /* kda_decode_commit: accepted count outside [0, K] */
} kda_status;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype;

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int kda_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char *kda_status_string(kda_status s);

/*
 * How this copy of the library was built.  KDA_BUILD_DEBUG_CHECKS is set in the
 * debug build (libkda_b200_debug.so, compiled with -DKDA_DEBUG=1): at the top of
 * every prefill kernel the indices that address global memory (chunk table
 * entries, sequence token ranges, record slots) are checked against their
 * buffers' extents, and a failed check makes the affected CTAs return before
 * their first access and the call's device error KDA_ERR_DEBUG_BOUNDS, instead of
 * an out-of-bounds access.  The release build (libkda_b200.so) has no checks.
 */
#define KDA_BUILD_DEBUG_CHECKS 1
int kda_build_flags(void);

/*
 * Bytes of device workspace that kda_fwd needs for these sizes.  The
 * tensor-core path stores, per 64-token chunk and head, the chunk's affine map
 * on the state (98,816 bytes: the state transition and offset, the output
 * read-out and offset, and the chunk's total decay) that the state pass consumes,
 * plus a 4-byte ready flag per record and a few KiB of progress counters for the
 * overlapped single-launch schedule.
 * When few (sequence, head) chains would leave most SMs idle, kda_fwd splits
 * each chain in time (see kda_fwd_segmented); the size returned here includes
 * room for the largest split the library would choose on a GPU of up to 192
 * SMs, so it does not depend on the current device.
 * Returns 0 for an invalid or unsupported combination.
 *   B, T      : fixed-length batch (B sequences of T tokens), or with
 *               num_seqs > 0 and packed input: B = 1, T = total tokens.
 *   num_seqs  : 0 for fixed-length input, else the number of packed sequences.
 */
size_t kda_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int dtype);

/*
 * Chunkwise prefill: runs the recurrence over every (sequence, head) from its
 * initial state and returns all outputs and the final states.
 *
 *   q, k     [B, T, H, d_k]  dtype      keys and queries used as given
 *   v        [B, T, H, d_v]  dtype
 *   g        [B, T, H, d_k]  fp32       log-decay; precondition g <= 0
 *                                       (the pages bound it to (-5, 0))
 *   beta     [B, T, H]       fp32       write strength
 *   h0       [N, H, d_k, d_v] fp32      initial states; NULL means zeros
 *   cu_seqlens [num_seqs + 1] int32     NULL for fixed-length input; otherwise
 *                                       packed sequence offsets (B must be 1,
 *                                       cu_seqlens[0] = 0, non-decreasing,
 *                                       cu_seqlens[num_seqs] = T).  Empty
 *                                       sequences are allowed (hT = h0).
 *   o        [B, T, H, d_v]  dtype      outputs; must not alias any input
 *   hT       [N, H, d_k, d_v] fp32      final states, NULL to skip.  hT == h0 is
 *                                       allowed (the update is then in place).
 *   workspace, ws_bytes                 device scratch of at least
 *                                       kda_fwd_workspace_size(...) bytes; its
 *                                       contents on entry do not matter.
 *   N = B for fixed-length input, N = num_seqs for packed input.
 *
 * The cu_seqlens preconditions are checked on the device; a violation makes
 * the call write no outputs and is reported by kda_get_last_device_error.
 * T = 0 (or B = 0) is a valid empty call that only copies h0 to hT.
 * On the tensor-core path the call picks its schedule itself from the SM count:
 * the number of time segments of the state pass (kda_fwd_segmented: split only
 * when N * H chains are too few to fill the GPU), and, for fixed-length input
 * without a split, whether both phases run as one overlapped launch
 * (kda_fwd_overlapped) or as two (kda_fwd_segmented with one segment; also taken
 * when the device refuses the overlapped launch).
 */
kda_status kda_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *h0, const int32_t *cu_seqlens,
                   int num_seqs, int B, int T, int H, int dk, int dv, int dtype, void *o,
                   float *hT, void *workspace, size_t ws_bytes, void *stream);

/*
 * The two phases of kda_fwd on the tensor-core path (bf16, d_k = d_v = 128),
 * exposed so callers can schedule or time them separately.  Calling
 * kda_fwd_intra and then kda_fwd_inter on the same stream and workspace is
 * exactly kda_fwd_segmented with one segment (and kda_fwd, where kda_fwd neither
 * splits nor overlaps: kda_fwd_plan_segments and kda_fwd_plan_overlap say which).
 * Other dtype / head-size combinations return
 * KDA_ERR_UNSUPPORTED_SHAPE (kda_fwd handles them in a single kernel).
 *
 * kda_fwd_intra: everything inside a chunk, in parallel over (chunk, head):
 *   validates cu_seqlens and lays out the chunks (packed input), then computes
 *   the in-chunk cumulative log-decay, the strictly-lower key-key block and its
 *   unit-triangular inverse, the delta-rule factors W and U, the decayed keys
 *   and queries, the masked query-key block and the chunk's total decay, and
 *   stores them in `workspace`.  Arguments as for kda_fwd.
 * kda_fwd_inter: the sequential pass over the chunks of every (sequence, head)
 *   with the state on chip: reads the records from `workspace`, writes o and hT.
 *   The size arguments must match the preceding kda_fwd_intra call.
 */
kda_status kda_fwd_intra(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const int32_t *cu_seqlens, int num_seqs, int B,
                         int T, int H, int dk, int dv, int dtype, void *workspace,
                         size_t ws_bytes, void *stream);
kda_status kda_fwd_inter(const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T,
                         int H, int dk, int dv, int dtype, void *o, float *hT, void *workspace,
                         size_t ws_bytes, void *stream);

/*
 * Prefill with an explicit time split of the state pass.  Source: the "Kimi K3"
 * field notes, panel "传固定状态片段" (pass fixed-size state fragments): each
 * worker summarises its stretch of the sequence as a cumulative transform plus
 * a state grown from zero, and the stretches are then combined in prefix order;
 * the same page's "FlashKDA / FLA" panel names the within-device form of this
 * context parallelism, which is what this entry point does.  It works because
 * every chunk's map on the state is affine, S -> P S + R.
 *
 * Each chain's chunks are cut into num_segments consecutive segments of
 * ceil(chunks / num_segments) chunks (trailing segments may be short or empty).
 * Pass 1 computes every segment's map [R | P] from zero / identity, a combine
 * kernel walks the segments in order in fp32 (S_{s+1} = P_s S_s + R_s) to get
 * each segment's starting state, and pass 2 reruns the segments from those
 * states, writing o and (from the last segment) hT.  num_segments = 1 is the
 * unsplit pass as two launches (kda_fwd_intra, then kda_fwd_inter), which is what
 * kda_fwd runs when it neither splits nor overlaps.  num_segments > 1 needs the tensor-core path
 * (bf16, d_k = d_v = 128), else KDA_ERR_UNSUPPORTED_SHAPE; at most 4,096.
 * The workspace must hold kda_fwd_segmented_workspace_size(..., num_segments)
 * bytes: the records plus N * H * num_segments * 192 KiB.
 * Other arguments and results as for kda_fwd.
 */
size_t kda_fwd_segmented_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                        int dtype, int num_segments);
/* The number of time segments kda_fwd chooses for these sizes on the current
 * device (1: no split; 0: invalid or unsupported sizes, or no device). */
int kda_fwd_plan_segments(int B, int T, int H, int dk, int dv, int num_seqs, int dtype);
kda_status kda_fwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                             int num_segments, void *o, float *hT, void *workspace,
                             size_t ws_bytes, void *stream);

/*
 * Prefill with both phases in ONE launch, overlapped in time (fixed-length input,
 * tensor-core path: bf16, d_k = d_v = 128).  The state pass of a chain is
 * sequential over its chunks, while the chunk records are independent; with few
 * chains the state pass occupies few SMs for a long time.  Here one block per SM
 * is launched: 2 * B * H of them run the state pass (64-column slices of each
 * (sequence, head) state) and every other block runs two workers of the record
 * kernel, which write the records in time order (chunk j of every chain before
 * chunk j + 1) and publish each through a flag in the workspace; a state block
 * waits (bounded, 1 s) for a record's flag before copying it in, and a record
 * worker starts a chunk only within a window of chunks (about 32 MiB of records)
 * ahead of that chain's state blocks, so the records are read back from L2.  Each
 * waits only for work that comes earlier in time order than what it holds, so the
 * blocks cannot deadlock; the launch is cooperative so that every block is
 * resident.  Results equal those of
 * kda_fwd_segmented with one segment up to the state pass's bf16 rounding (the two
 * schedules slice the state differently), and are checked against the oracle at
 * the same tolerance.
 *
 * Needs 2 * B * H below the device's SM count (else KDA_ERR_UNSUPPORTED_SHAPE);
 * packed input is not supported (no cu_seqlens argument).  Workspace: at least
 * kda_fwd_segmented_workspace_size(B, T, H, 128, 128, 0, dtype, 1) bytes (which
 * kda_fwd_workspace_size covers).  A record that is never published makes the
 * state blocks give up after the bounded wait: the call's device error becomes
 * KDA_ERR_DEVICE_TIMEOUT.  Other arguments and results as for kda_fwd.
 */
kda_status kda_fwd_overlapped(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *h0, int B, int T, int H, int dk,
                              int dv, int dtype, void *o, float *hT, void *workspace,
                              size_t ws_bytes, void *stream);
/* 1 if kda_fwd runs the overlapped single launch for these sizes on the current
 * device, else 0 (also for invalid sizes, packed input or no device). */
int kda_fwd_plan_overlap(int B, int T, int H, int dk, int dv, int num_seqs, int dtype);

/*
 * kda_fwd that also stores the state at fixed token intervals, for prefix caching
 * (a later call resumes from a stored state as its h0).  The state is the one
 * after a whole number of tokens; checkpoints sit on the 64-token chunk
 * boundaries, so ckpt_every must be a positive multiple of 64.
 *
 * For sequence n of length L_n and head h, checkpoint c = 0 .. L_n / ckpt_every - 1
 * (integer division) is the state after the sequence's first (c + 1) * ckpt_every
 * tokens, stored fp32 at
 *     ckpts[((first_n + c) * H + h) * d_k * d_v ...],   [d_k][d_v] row-major,
 *     first_n = sum over m < n of L_m / ckpt_every,
 * i.e. ckpts is [num_checkpoints, H, d_k, d_v] with the checkpoints of each sequence
 * together and in token order.  ckpt_capacity is the number of checkpoint slots
 * (the first dimension of ckpts).  For fixed-length input it must be at least
 * B * (T / ckpt_every), else KDA_ERR_INVALID_ARG; for packed input the lengths
 * live on the device, so a checkpoint past the capacity is not written and the
 * call's device error becomes KDA_ERR_CHECKPOINT_CAPACITY.
 *
 * Tensor-core path only (bf16, d_k = d_v = 128), else KDA_ERR_UNSUPPORTED_SHAPE.
 * ckpts must be 16-byte aligned (KDA_ERR_MISALIGNED) and must not overlap any
 * other argument.  Workspace, o, hT and the time-split policy as for kda_fwd; o
 * and hT are bitwise those of kda_fwd.
 *
 * Source: the "Kimi K3" open-weights field notes, panel "目标模型太大，缓存和草稿都必须
 * 理解 KDA" (a prefix cache must restore the KDA recurrent state at the same token
 * boundary as the attention cache), and the API card's 256-token shortest cached
 * prefix; the stored state is the recurrence's S_t (panel "KDA 单头递归").
 */
kda_status kda_fwd_checkpointed(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                                void *o, float *hT, int ckpt_every, float *ckpts,
                                long long ckpt_capacity, void *workspace, size_t ws_bytes,
                                void *stream);

/*
 * One decode step: every (sequence, head) consumes one token and updates its
 * state in place (the recurrence above with T = 1).
 *
 *   q, k [N, H, d_k] dtype;  v [N, H, d_v] dtype;  g [N, H, d_k] fp32;
 *   beta [N, H] fp32;  S [N, H, d_k, d_v] fp32, read and overwritten;
 *   o [N, H, d_v] dtype, the read of the updated state.
 * Each state is read from HBM once and written once.  N = 0 is a no-op.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float *S, void *o, int N, int H, int dk,
                           int dv, int dtype, void *stream);

/*
 * Context parallelism across devices: one sequence batch split in time over
 * `world` ranks (rank r holds tokens [r T_local, (r + 1) T_local) of every
 * sequence).  Source: the "Kimi K3" field notes, panel "传固定状态片段" (pass
 * fixed-size state fragments): each rank summarises its stretch as a cumulative
 * transform plus a state grown from zero, one all-gather exchanges those
 * fixed-size summaries, and each rank combines the summaries of the ranks before it
 * in prefix order to get its starting state.  This works because every chunk's map
 * on the state is affine, S -> P S + R (panel "KDA 单头递归" unrolled over a chunk).
 *
 *   1. kda_cp_local_map: the intra-chunk pass over the local tokens, then the map
 *      pass over the whole local stretch: seg_map [B, H, d_k, 2 d_v] fp32 = [R | P]
 *      per (sequence, head) -- R the local final state from zero, P the linear part.
 *      The chunk records stay in `workspace` for step 3.
 *   2. (caller) all-gather seg_map over the ranks, in rank order, into
 *      maps [world, B, H, d_k, 2 d_v] -- 128 KiB per (sequence, head) per rank.
 *   3. kda_cp_finish: S_in = fold over ranks 0 .. rank-1 of S <- P_s S + R_s from h0
 *      (the sequences' initial states, NULL: zero; the same on every rank), written
 *      to s_in [B, H, d_k, d_v]; then the state pass from S_in over the local
 *      records, writing the local outputs o [B, T_local, H, d_v] and hT, the state
 *      after the local stretch (on the last rank: the sequences' final states).
 *      maps may be NULL on rank 0.
 * Fixed-length input and the tensor-core path only (bf16, d_k = d_v = 128), else
 * KDA_ERR_UNSUPPORTED_SHAPE.  The workspace must hold kda_cp_workspace_size bytes
 * and be the same buffer, unchanged, in steps 1 and 3.  s_in must not alias h0, o
 * or hT.  Alignment as kda_fwd; seg_map, maps and s_in 16 bytes.
 */
size_t kda_cp_workspace_size(int B, int T_local, int H, int dk, int dv, int dtype);
kda_status kda_cp_local_map(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, int B, int T_local, int H, int dk, int dv,
                            int dtype, float *seg_map, void *workspace, size_t ws_bytes,
                            void *stream);
kda_status kda_cp_finish(const float *maps, int rank, int world, const float *h0, float *s_in,
                         int B, int T_local, int H, int dk, int dv, int dtype, void *o,
                         float *hT, void *workspace, size_t ws_bytes, void *stream);

/*
 * Backward pass: the gradient of a loss L through kda_fwd.  Given grad_o = dL/do and
 * grad_hT = dL/dhT (NULL: zero), writes dL/dq, dL/dk, dL/dv (dtype of q, k, v),
 * dL/dg, dL/dbeta (fp32) and dL/dh0 (fp32, NULL to skip).  Same inputs, layouts,
 * packed-sequence rules and alignment as kda_fwd, except that g and grad_o must be
 * 16-byte aligned (rows are staged by 16-byte copies); grad_o [B, T, H, d_v] has the
 * dtype of q; grad_hT, grad_h0 [N, H, d_k, d_v].  No gradient buffer may alias an
 * input.  The workspace must hold kda_bwd_workspace_size(...) bytes.
 *
 * What it computes is the chain rule through the recurrence (panel "KDA 单头递归"),
 * token by token from the last to the first, with G = dL/dS_t, S' = Diag(exp g_t)
 * S_{t-1}, u = S'^T k and delta = v - u:
 *     G += q do^T;  dq = S_t do;  w = G delta;  dbeta = k . w;  dv = beta G^T k;
 *     dk = beta w - S' dv;  G' = G - k dv^T;  dg_i = sum_j S'_ij G'_ij;
 *     G = Diag(exp g) G';  and dh0 = G after the first token.
 * The source pages name the training kernel ("FlashKDA / FLA" panel) but give no
 * formulas for it; this is the gradient of the recurrence they print, applied in fp32
 * on CUDA cores per (sequence, head) and 16 value columns, the slices of a chain (or of
 * a segment of it) one thread-block cluster, states recomputed from checkpoints.
 *
 * Two schedules (kda_bwd_segmented chooses explicitly):
 *   per chain:  each chain walked whole, from h0 and dL/dhT; every dtype, head size
 *               and the packed layout.  Workspace: the state every 64 tokens of every
 *               (sequence, head) (d_k d_v / 16 bytes per token-head) plus 8 states per
 *               (sequence, head).  The gradients stored in fp32 match an fp64
 *               evaluation to about 1e-7.
 *   segmented:  (bf16, d_k = d_v = 128, fixed-length input, grad_q and grad_k
 *               16-byte aligned) the chain cut into segments of whole 64-token chunks,
 *               all run at once.  A segment's starting state comes from the tensor-core
 *               forward (kda_fwd's records and state pass, with a checkpoint at every
 *               segment start), its ending gradient from the chunk-level chain
 *               dL/dS_in = Diag(exp G_C) dL/dS_out + M'^T dL/dS_out + Q'^T dO run by the
 *               same state pass backwards over the chunks (reversed records); both carry
 *               the bf16 records' rounding, so every gradient is held to the bf16
 *               prefill bound (rel-L2 <= 1e-2).  grad_q and grad_k serve as scratch for
 *               the two state passes' outputs before they receive the gradients.
 *               Workspace: the chunk records twice (forward and reversed, 1,544 bytes
 *               per token-head each at d = 128), a state and a state gradient per
 *               segment boundary, the 64-token checkpoints as above and 8 states per
 *               (sequence, head, segment).
 * kda_bwd takes the segmented schedule whenever it applies and some cut leaves at least
 * two segments: one chunk per segment, or the fewest chunks (a power of two dividing
 * the chunks per sequence) that keep (sequences x heads x segments) <= 1024.
 */
size_t kda_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int dtype);
kda_status kda_bwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                   int B, int T, int H, int dk, int dv, int dtype, const void *grad_o,
                   const float *grad_hT, void *grad_q, void *grad_k, void *grad_v,
                   float *grad_g, float *grad_beta, float *grad_h0, void *workspace,
                   size_t ws_bytes, void *stream);

/*
 * kda_bwd with the schedule chosen by the caller: num_segments = 0 as kda_bwd, 1 the
 * per-chain pass (any input kda_bwd takes), n >= 2 the segmented pass with n segments
 * per sequence (n must divide ceil(T / 64); bf16, d = 128, fixed-length input, else
 * KDA_ERR_UNSUPPORTED_SHAPE; grad_q, grad_k 16-byte aligned, else
 * KDA_ERR_MISALIGNED).  The workspace must hold
 * kda_bwd_segmented_workspace_size(..., num_segments) bytes (0 when the request cannot
 * be met).
 */
size_t kda_bwd_segmented_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                        int dtype, int num_segments);
/* The segments per sequence kda_bwd uses for these sizes (1: the per-chain pass; it
 * may still take the per-chain pass when the alignment rule above is not met); 0 on
 * invalid sizes. */
int kda_bwd_plan_segments(int B, int T, int H, int dk, int dv, int num_seqs, int dtype);
kda_status kda_bwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                             const void *grad_o, const float *grad_hT, void *grad_q, void *grad_k,
                             void *grad_v, float *grad_g, float *grad_beta, float *grad_h0,
                             int num_segments, void *workspace, size_t ws_bytes, void *stream);

/*
 * Speculative decoding: verify K drafted tokens per sequence, then commit the
 * accepted prefix.  Source: the "Kimi K3" open-weights field notes, panel
 * "目标模型太大，缓存和草稿都必须理解 KDA": with a draft model the KDA recurrent
 * state must follow only the tokens the target model accepts -- a rejected draft
 * must not remain in the state -- and K3 keeps the projected inputs of the drafted
 * tokens and replays the accepted ones on chip instead of storing a state per
 * drafted token.  The recurrence is the one above (panel "KDA 单头递归"), token by
 * token in draft order.
 *
 * kda_decode_verify: for every (sequence n, head h), run the K drafted tokens from
 *   the state S and write their K outputs; S is only read.
 *     q, k, g [N, K, H, d_k] dtype / fp32;  v [N, K, H, d_v] dtype;
 *     beta [N, K, H] fp32;  S [N, H, d_k, d_v] fp32 (read);
 *     o [N, K, H, d_v] dtype: o[n, t] is the read of the state after draft
 *     tokens 0..t -- what K chained kda_decode_step calls would return.
 * kda_decode_commit: for every (sequence n, head h), replay the first accepted[n]
 *   drafted tokens (the same k, v, g, beta the verify call saw) from S and write
 *   the resulting state to S in place: S becomes the state after the accepted
 *   prefix, as if only those tokens had been decoded.  accepted is a DEVICE array
 *   of N int32 counts in [0, K] (typically written by the sampler on the GPU);
 *   accepted[n] = 0 leaves sequence n's state untouched.  A count outside [0, K]
 *   leaves that sequence's state untouched and makes the call's device error
 *   KDA_ERR_BAD_ACCEPTED (see kda_get_last_device_error).
 * 1 <= K <= 16 (K = 0 or N = 0 is a no-op; K > 16 returns KDA_ERR_INVALID_ARG).
 * Alignment: S 16 bytes, everything else its element size.  o must not alias an
 * input.  Cost: verify reads each state once; commit reads and writes it once --
 * against K reads and K writes for K single decode steps.
 */
kda_status kda_decode_verify(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *S, void *o, int N, int K, int H,
                             int dk, int dv, int dtype, void *stream);
kda_status kda_decode_commit(const void *k, const void *v, const float *g, const float *beta,
                             const int32_t *accepted, float *S, int N, int K, int H, int dk,
                             int dv, int dtype, void *stream);

/*
 * Allocation-free prefill.  The source pages have no counterpart to this entry
 * point: it is a convenience of this library, not part of the method.
 *
 * Some callers cannot allocate device memory on the call path: code that a
 * host framework or plugin interface hands only its input and output buffers,
 * with no way to ask for scratch space, and code whose device-memory budget is
 * fixed up front so that a per-call allocation (and the chance of it failing
 * mid-request) is not allowed.  kda_fwd needs a caller-provided workspace; this
 * variant instead uses one scratch array compiled into the library -- a
 * file-scope __device__ array of KDA_NOALLOC_SCRATCH_BYTES (32 MiB) that every
 * GPU which loads the library keeps until the process exits.  It calls no
 * cudaMalloc or cudaFree and no allocating library routine.
 *
 * Arguments and results are those of kda_fwd without the workspace arguments.
 * Only the tensor-core path is offered (bf16, d_k = d_v = 128); other dtypes or
 * head sizes return KDA_ERR_UNSUPPORTED_SHAPE.
 *
 *   - Size limit: this variant never splits the state pass in time, so its
 *     scratch need is kda_fwd_segmented_workspace_size(B, T, H, 128, 128,
 *     num_seqs, KDA_DTYPE_BF16, 1); that must not exceed
 *     KDA_NOALLOC_SCRATCH_BYTES, otherwise the
 *     call returns KDA_ERR_EXCEEDS_STATIC_SCRATCH and launches nothing.  32 MiB
 *     holds 339 (64-token chunk, head) records, e.g. B = 1, H = 8, T = 2,688.
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it for that
 *     device's current CUDA context; a new context on the device (after
 *     cudaDeviceReset, for instance) gets a fresh lookup on its first call, and a
 *     lookup that fails is not cached (the call returns KDA_ERR_CUDA and the next
 *     call tries again).  Make the first call on each device, and in each new
 *     context, before any stream capture begins.
 *   - Sharing: every call on a device uses the same array, which keeps whatever
 *     the previous call left in it.  Nothing in it has to start at zero, because
 *     each call writes every scratch byte it later reads.  Calls whose work
 *     overlaps on the GPU (issued on different streams, or from different host
 *     threads without ordering) race on the array and corrupt each other's
 *     results: order them on one stream or with events.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
kda_status kda_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, const int32_t *cu_seqlens,
                           int num_seqs, int B, int T, int H, int dk, int dv, int dtype, void *o,
                           float *hT, void *stream);

/*
 * Synchronises `stream`, then reads and clears the library's device error word
 * (cu_seqlens violations, bounded waits that gave up, checkpoints past the
 * capacity, debug bounds checks, accepted counts out of range).  Returns KDA_OK,
 * KDA_ERR_BAD_SEQLENS, KDA_ERR_DEVICE_TIMEOUT, KDA_ERR_CHECKPOINT_CAPACITY,
 * KDA_ERR_DEBUG_BOUNDS, KDA_ERR_BAD_ACCEPTED or KDA_ERR_CUDA.
 */
kda_status kda_get_last_device_error(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_H */
