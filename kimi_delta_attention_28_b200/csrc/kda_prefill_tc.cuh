// kda_prefill_tc.cuh -- chunkwise KDA prefill on tensor cores, bf16 q/k/v, d_k = d_v = 128.
//
// The recurrence (single head, "Kimi K3" open-weights field notes, panel
// "KDA 单头递归"):  S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t.  Over a chunk of C tokens with inclusive cumulative log-decay
// G_r (per key channel), unrolling the recurrence gives the exact chunk form
//
//   A_ri  = b_r sum_c k_rc k_ic exp(G_rc - G_ic)      (i < r, strictly lower)
//   [W|U] = (I + A)^-1 Diag(b) [K * exp G | V]
//   Delta = U - W S_in                                (per-token delta-rule errors)
//   O     = (Q * exp G) S_in + [i <= r](sum_c q_rc k_ic exp(G_rc - G_ic)) Delta
//   S_out = Diag(exp G_C) S_in + (K * exp(G_C - G))^T Delta
//
// Kernel 1 (kda_tc_prep_kernel) computes every chunk-local quantity, in parallel
// over (chunk, head) items (persistent CTAs that load the next item while finishing
// the current one): the log-decay cumsum; the key-key and query-key blocks with the
// pairwise decays factored through 16-token sub-tile reference rows so no factor
// overflows (the same page's panel "g ∈ (-5, 0)" bounds a 16-token decay by e^-80);
// T' = (I + A)^-1 Diag(b) by blocked forward substitution (fp32 inverses of the
// 16x16 diagonal blocks, warp-level tensor-core products elsewhere); [W|U] = T' [K *
// exp G | V] and from it the chunk's affine map on the state (below) on tcgen05,
// one record per (chunk, head).
// Kernel 2 (kda_tc_state_kernel) walks the chunks of each (sequence, head) in
// order with the fp32 state on chip, split over 32- or 64-column slices of the
// state (state columns evolve independently).  Its warps are specialised (state
// update, tcgen05 issue, output, bulk-copy producer) and hand off through
// mbarriers, so the loop-carried path per chunk is one tcgen05 product plus the
// register update of the state; the outputs and copies run beside it.
// kda_tc_fused_kernel runs both in one cooperative launch for few long chains: state
// blocks consume each record as soon as prep workers in the other blocks publish it.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace tc {

constexpr int D = 128;          // head size (d_k = d_v)
constexpr int C = 64;           // chunk length
constexpr int ST = 16;          // sub-tile length for the decay reference rows
constexpr int NST = C / ST;     // sub-tiles per chunk
// A 4-D tensor copy (tma_load_4d) with an L2 eviction-priority hint (`policy`, from
// l2_evict_first): for data read exactly once, so that it does not displace data
// still to be read.
KDA_DEVINL void tma_load_4d_hint(void *smem_dst, const CUtensorMap *tm, int c0, int c1, int c2,
                                 int c3, uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;\n"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1),
          "r"(c2), "r"(c3), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// An L2 cache policy that marks every access it is given as evict-first.
KDA_DEVINL uint64_t l2_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
    return p;
}

// Largest total decay of a chunk (log2 units, per channel) for which the prep uses
// one reference row and whole-chunk tensor-core products: factors up to 2^120 stay
// inside the bf16 / fp32 range (2^127) with room for |k| <= 1.
constexpr float kDenseSpan = 120.f;

// Per (chunk, head) record, written by kernel 1 and read by kernel 2: the
// chunk's affine map.  With W, U, Kt = K*exp(G_C - G), Qg = Q*exp(G) and the
// masked query-key block Aqk, a chunk takes the state S_in to
//   S_out = Diag(exp G_C) S_in + M' S_in + R,   M' = -Kt^T W,  R = Kt^T U
//   O     = Q' S_in + O0,                      Q' = Qg - Aqk W,  O0 = Aqk U
// The four matrices use the core-matrix layout (core_off): 8-column chunks
// outermost, rows inside, 16 bytes per (row, chunk).  A warp whose lanes hold
// consecutive rows writes 512 contiguous bytes per 16-byte store, the layout is
// the tensor core's non-swizzled K-major operand layout (M' and Q' are A
// operands of the state pass), and any 8-column-aligned slice of R or O0 is one
// contiguous block.
constexpr int REC_M = 0;                     // M'        [D][D] bf16, core_off(D, ...)
constexpr int REC_QP = REC_M + D * D * 2;    // Q'        [C][D] bf16, core_off(C, ...)
constexpr int REC_GC = REC_QP + C * D * 2;   // exp(G_C)  [D] fp32
constexpr int REC_SHARED = REC_GC + D * 4;   // bytes every column slice reads (49,664)
constexpr int REC_R = REC_SHARED;            // R         [D][D] bf16, core_off(D, ...)
constexpr int REC_O0 = REC_R + D * D * 2;    // O0        [C][D] bf16, core_off(C, ...)
constexpr int REC_BYTES = REC_O0 + C * D * 2;  // 98,816
// Kt and Qg pass through the R and O0 areas of the record (swizzled layouts)
// before those are written: kernel 1 needs them after its shared memory has been reused.
constexpr int REC_KT_SCRATCH = REC_R;
constexpr int REC_QG_SCRATCH = REC_O0;
static_assert(REC_BYTES % 256 == 0 && REC_SHARED % 16 == 0 && REC_O0 % 16 == 0, "alignment");

// Byte offset of bf16 element (r, c) of a [rows][D] matrix in the core-matrix layout.
KDA_DEVINL int core_off(int rows, int r, int c) {
    return (c >> 3) * (rows * 16) + r * 16 + ((c & 7) << 1);
}

// Byte offset of element (r, c) of a [rows][128] bf16 tile stored as two planes
// (columns 0-63, then 64-127), each with 128-byte rows and the 16-byte chunks of
// row r XOR-permuted by (r & 7): the K-major (or N-major) 128-byte-swizzled operand
// layout the tcgen05 tensor core reads from shared memory (8-row groups 1024
// bytes apart).
KDA_DEVINL int umma_k128(int rows, int r, int c) {
    return (c >> 6) * (rows * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

struct ChunkLoc {
    int t0;    // first token (flattened over the batch / packed sequences)
    int len;   // tokens in this chunk, 1..C
};

constexpr int ERR_TIMEOUT_BIT = 2;
constexpr int ERR_CKPT_BIT = 4;     // a state checkpoint fell past the caller's capacity
constexpr int ERR_BOUNDS_BIT = kErrBoundsBit;   // debug builds: an index failed its bounds check

// ---------------------------------------------------------------------------
// Varlen chunk map: validates cu_seqlens and lays out each sequence's chunks.
// One block.  hdr[0] = 1 when valid; seq_off[n] = first chunk of sequence n.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) kda_chunk_map_kernel(const int *__restrict__ cu, int N,
                                                             int T, int *hdr, int *seq_off,
                                                             ChunkLoc *chunks, int max_chunks,
                                                             int *err_word, int err_code) {
    __shared__ int s_bad;
    __shared__ int s_scan[1024];
    const int tid = threadIdx.x;
    if (tid == 0) s_bad = (cu[0] != 0 || cu[N] != T) ? 1 : 0;
    __syncthreads();
    for (int n = tid; n < N; n += blockDim.x)
        if (cu[n + 1] < cu[n]) s_bad = 1;
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            hdr[0] = 0;
            hdr[1] = 0;
            atomicOr(err_word, err_code);
        }
        return;
    }
    // Each thread owns a contiguous range of sequences; block-scan the counts.
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
    int cnt = 0;
    for (int n = n0; n < n1; ++n) cnt += (cu[n + 1] - cu[n] + C - 1) / C;
    s_scan[tid] = cnt;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        int x = (tid >= off) ? s_scan[tid - off] : 0;
        __syncthreads();
        s_scan[tid] += x;
        __syncthreads();
    }
    if constexpr (KDA_DEBUG) {   // valid offsets give at most T / C + N chunks
        if (s_scan[blockDim.x - 1] > max_chunks) {
            if (tid == 0) {
                hdr[0] = 0;
                hdr[1] = 0;
                atomicOr(err_word, ERR_BOUNDS_BIT);
            }
            return;
        }
    }
    int base = s_scan[tid] - cnt;
    for (int n = n0; n < n1; ++n) {
        seq_off[n] = base;
        const int L = cu[n + 1] - cu[n];
        for (int j = 0; j * C < L; ++j) {
            chunks[base + j].t0 = cu[n] + j * C;
            chunks[base + j].len = min(C, L - j * C);
        }
        base += (L + C - 1) / C;
    }
    if (tid == blockDim.x - 1) {
        seq_off[N] = s_scan[tid];
        hdr[1] = s_scan[tid];
        hdr[0] = 1;
    }
}

// ---------------------------------------------------------------------------
// Kernel 1: intra-chunk transform.  Persistent: grid = min(items, 2 per SM) CTAs of
// 256 threads; CTA b takes the (chunk, head) items b, b + gridDim.x, ... and loads
// each item's inputs while the previous item's last products and epilogues run, into
// the tiles those phases have just released.
// ---------------------------------------------------------------------------
constexpr int LDA = C + 8;      // padded bf16 row stride of the 64x64 blocks (144 B)

// The six sub-tile pairs (a, b), b < a, of a 64-token chunk.
__constant__ int2 kPairs[6] = {{1, 0}, {2, 0}, {3, 0}, {2, 1}, {3, 1}, {3, 2}};

struct PrepSmem {
    // Five 16 KB tiles, reused across phases.  Every bf16 tile uses the tensor core's
    // K-major 128-byte-swizzled layout (umma_k128: two 64-column planes of 128-byte
    // rows), which is also the layout the tensor-memory-access engine writes with its
    // 128-byte swizzle, and in which ldmatrix reads 8 rows of a column chunk without
    // bank conflicts.  An item's inputs arrive as: g rows 0-31 in ka and rows 32-63 in
    // xk (fp32, 512-byte rows); k in qa, q in kb; V in xv.
    //   ka: g (rows 0-31); k*exp(G_r - G_ref(a)); then T' = (I + A)^-1 Diag(b) (first 8 KB)
    //   qa: raw k; q*exp(G_r - G_ref(a)); then, with kb, [W|U] (four planes)
    //   kb: raw q; k*exp(G_ref(a) - G_r)
    //   xk: g (rows 32-63); K*exp(G); then Kt
    //   xv: V; then Qg.  xk and xv are contiguous: together they are the N = 256 right
    //       operand [K*exp G | V] of the [W|U] product.
    uint8_t ka[C * D * 2], qa[C * D * 2], kb[C * D * 2], xk[C * D * 2], xv[C * D * 2];
    __nv_bfloat16 akkn[C * LDA];   // -b_r A_ri, sub-tile blocks b < a (bf16)
    uint8_t aqk[C * C * 2];        // masked query-key block, umma_k128 plane (bf16)
    __nv_bfloat16 taa[NST][ST * (ST + 8)];  // (I + A_aa)^-1, bf16
    float mfac[6][D];              // exp(G_ref(a) - G_ref(b)) per pair and channel
    union {
        struct {
            float tot[NST][D];     // sub-tile decay totals   (log2 units)
            float ref[NST][D];     // sub-tile-local G at the reference row
        } p1;
        float akd[NST][ST][ST];    // b_r A_ri inside the diagonal sub-tile blocks
    } u;
    float beta[C];
    uint64_t mma_bar;              // tcgen05 completion barrier
    uint64_t ld_bar[4];            // input loads: g rows 0-31, g rows 32-63, k and q, V
    uint32_t tmem_slot;            // tensor-memory base address (written by tcgen05.alloc)
};

// Arguments of kernel 1 besides the tensor maps.
struct PrepArgs {
    const float *beta;
    int T, H, cps, slots;
    const int *hdr;
    const ChunkLoc *chunks;
    uint8_t *recs;
    int *err_word;
    // Overlapped schedule (one launch with the state pass, fixed-length input only):
    // items in time order -- chunk j of every (sequence, head) before chunk j + 1 --
    // and a flag per record, ready[chunk * H + head], set (release, GPU scope) once
    // the record is complete.  Null: items in sequence order, no flags.
    int *ready;
    int nseq;
    int nstate;   // overlapped schedule: state blocks before the prep blocks
    // Overlapped schedule: chunks each state CTA has started copying in (2 CTAs per
    // chain, column tile fastest); a worker starts the item of chunk j of a chain only
    // once both of the chain's CTAs have reached chunk j - window, so the records in
    // flight between the two roles stay within L2.  Null: no limit.
    const int *progress;
    int window;
};
constexpr int kPrepThreads = 256;   // one prep worker: 8 warps

// Progress counters of the state CTAs: one per 128-byte line, so that pollers of
// one chain do not contend with the stores of another.
constexpr int kProgStride = 32;
// Wait until both state CTAs of a chain have started chunk `need` (bounded; polled
// about once a microsecond: the counters advance once per chunk period).
KDA_DEVINL bool progress_wait_bounded(const int *prog2, int need) {
    auto reached = [&]() {
        int a, b;
        asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];\n" : "=r"(a) : "l"(prog2) : "memory");
        asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];\n"
                     : "=r"(b) : "l"(prog2 + kProgStride) : "memory");
        return a >= need && b >= need;
    };
    if (reached()) return true;
    const uint64_t t0 = global_timer_ns();
    while (!reached()) {
        __nanosleep(1000);
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// One prep worker: `kPrepThreads` threads with their own PrepSmem, whose tmem_slot
// holds the worker's 2D tensor-memory columns (allocated by the caller), walking
// items worker, worker + nworkers, ...
// OVERLAP = false: the standalone kernel, one worker per block (barrier 0).
// OVERLAP = true: two workers per block of the fused kernel after its p.nstate state
// blocks (worker w = threadIdx.x / 256 on named barrier 1 + w), with the overlapped
// schedule's item order, flags and window.  The indices are derived from the special
// registers where they are used rather than held in registers through the item loop
// (the standalone kernel's register budget is exactly full).
template <bool OVERLAP>
KDA_DEVINL void prep_worker(const CUtensorMap &tm_q, const CUtensorMap &tm_k,
                            const CUtensorMap &tm_v, const CUtensorMap &tm_g, const PrepArgs &p,
                            PrepSmem &sm) {
    const int tid = OVERLAP ? (int)(threadIdx.x % kPrepThreads) : (int)threadIdx.x;
    const int bar = OVERLAP ? 1 + (int)(threadIdx.x / kPrepThreads) : 0;
    const int worker = OVERLAP ? 2 * ((int)blockIdx.x - p.nstate) + (int)(threadIdx.x / kPrepThreads)
                               : (int)blockIdx.x;
    const int nworkers = OVERLAP ? 2 * ((int)gridDim.x - p.nstate) : (int)gridDim.x;
    // the worker's barriers: the block's own (barrier 0, immediate forms) when it is
    // alone in its block, else its named barrier
    auto cta_sync = [&]() {
        if constexpr (OVERLAP) bar_sync(bar, kPrepThreads);
        else __syncthreads();
    };
    auto cta_and = [&](bool x) {
        if constexpr (OVERLAP) return bar_and(bar, kPrepThreads, x);
        else return __syncthreads_and(x) != 0;
    };
    auto cta_or = [&](bool x) {
        if constexpr (OVERLAP) return bar_or(bar, kPrepThreads, x);
        else return __syncthreads_or(x) != 0;
    };
    const float *__restrict__ beta = p.beta;
    const int T = p.T, H = p.H, cps = p.cps, slots = p.slots;
    const int *__restrict__ hdr = p.hdr;
    const ChunkLoc *__restrict__ chunks = p.chunks;
    uint8_t *__restrict__ recs = p.recs;
    int *err_word = p.err_word;
    const int lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    if (chunks && !hdr[0]) return;
    const int items = (chunks ? min(hdr[1], slots) : slots) * H;
    if (worker >= items) return;
    const uint32_t s_ka = smem_u32(sm.ka), s_qa = smem_u32(sm.qa), s_kb = smem_u32(sm.kb);

    struct Item {
        int t0, len, h;
        int tl, b;         // the chunk's token and batch coordinates in the tensor maps
        int idx;           // record index: chunk * H + head
        uint8_t *rec;
    };
    const bool time_order = OVERLAP && !chunks;
    auto locate = [&](int item) {
        Item it;
        int cid;
        if (time_order) {
            const int per = p.nseq * H, j = item / per, r = item % per;
            cid = (r / H) * cps + j;
            it.h = r % H;
        } else {
            cid = item / H;
            it.h = item % H;
        }
        if (chunks) {
            it.t0 = chunks[cid].t0;
            it.len = chunks[cid].len;
            it.tl = it.t0;
            it.b = 0;
        } else {
            const int n = cid / cps, j = cid % cps;
            it.t0 = n * T + j * C;
            it.len = min(C, T - j * C);
            it.tl = j * C;
            it.b = n;
        }
        it.idx = cid * H + it.h;
        it.rec = recs + (size_t)it.idx * REC_BYTES;
        return it;
    };
    // Input loads by the tensor-memory-access engine (one thread issues them), in four
    // groups that complete on their own barriers and are issued as the previous item's
    // last phases release the tiles:
    //   ld_bar[0]: g rows 0-31 -> ka      ld_bar[1]: g rows 32-63 -> xk  (fp32 rows)
    //   ld_bar[2]: k -> qa, q -> kb       ld_bar[3]: V -> xv  (two 128B-swizzled planes)
    // Rows past the end of the tensor (fixed-length input: past T) arrive as zeros;
    // rows past the end of a packed sequence hold the next sequence's tokens and are
    // neutralised in P1: their g counts as zero and their beta is zero, so they neither
    // decay nor write the state.  beta comes by 4-byte cp.async beside k and q.
    uint32_t pend = 0, pend_par = 0;   // load groups in flight and the parity each completes
    // overlapped schedule: the inputs are read once, so they go through L2 as
    // evict-first and leave it to the records in flight between the two roles
    auto load = [&](void *dst, const CUtensorMap *tm, int c0, int c1, int c2, int c3, uint64_t *b) {
        if constexpr (OVERLAP) tma_load_4d_hint(dst, tm, c0, c1, c2, c3, b, l2_evict_first());
        else tma_load_4d(dst, tm, c0, c1, c2, c3, b);
    };
    auto issue = [&](int grp, const Item &it, uint32_t par) {
        if (tid == 0) {
            uint64_t *bar = &sm.ld_bar[grp];
            fence_proxy_async_smem();   // earlier generic accesses of the tile come first
            if (grp < 2) {
                mbar_arrive_expect_tx(bar, 32 * D * 4);
                load(grp ? sm.xk : sm.ka, &tm_g, 0, it.h, it.tl + 32 * grp, it.b, bar);
            } else if (grp == 2) {
                mbar_arrive_expect_tx(bar, 2 * C * D * 2);
#pragma unroll
                for (int pl = 0; pl < 2; ++pl) {
                    load(sm.qa + pl * C * 128, &tm_k, 64 * pl, it.h, it.tl, it.b, bar);
                    load(sm.kb + pl * C * 128, &tm_q, 64 * pl, it.h, it.tl, it.b, bar);
                }
            } else {
                mbar_arrive_expect_tx(bar, C * D * 2);
#pragma unroll
                for (int pl = 0; pl < 2; ++pl)
                    load(sm.xv + pl * C * 128, &tm_v, 64 * pl, it.h, it.tl, it.b, bar);
            }
        }
        if (grp == 2) {
            if (tid < C) {
                const bool in = tid < it.len;
                cp_async4(&sm.beta[tid], in ? beta + (size_t)(it.t0 + tid) * H + it.h : beta,
                          in ? 4 : 0);
            }
            cp_async_commit();
        }
        pend |= 1u << grp;
        pend_par = (pend_par & ~(1u << grp)) | ((par & 1u) << grp);
    };
    auto wait_ld = [&](int grp) {
        const bool done = mbar_wait_bounded(&sm.ld_bar[grp], (pend_par >> grp) & 1u);
        if (done) pend &= ~(1u << grp);
        return done;
    };

    if constexpr (KDA_DEBUG) {   // every item this CTA will take: a chunk of 1..C tokens
        const long long ntok = chunks ? (long long)T : (long long)(slots / max(cps, 1)) * T;
        bool bad = false;
        for (int item = worker + tid * nworkers; item < items; item += kPrepThreads * nworkers) {
            const Item it = locate(item);
            bad |= it.len < 1 || it.len > C || it.t0 < 0 || (long long)it.t0 + it.len > ntok ||
                   item / H >= slots;
        }
        if (cta_or(bad)) {
            if (tid == 0) atomicOr(err_word, ERR_BOUNDS_BIT);
            return;
        }
    }
    if (tid == 0) {
        mbar_init(&sm.mma_bar, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&sm.ld_bar[i], 1);
        fence_mbar_init();
    }
    // the query-key block is read whole by the tensor core: its upper blocks stay zero
    if (tid < 6 * ST * 2) {
        const int p = tid / (ST * 2), rr = (tid / 2) % ST, half = tid & 1;
        const int ba = kPairs[p].y, bb = kPairs[p].x;   // block (row ba, column bb), bb > ba
        *reinterpret_cast<uint4 *>(sm.aqk + umma_k128(C, ba * ST + rr, bb * ST + half * 8)) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t mma_phase = 0;   // completions of mma_bar so far
    uint32_t ld_phase = 0;    // items whose loads have been consumed
    bool ok = true;
    cta_sync();   // barrier initialisation is visible to every thread

    Item cur = locate(worker);
    for (int grp = 0; grp < 4; ++grp) issue(grp, cur, 0);

    for (int item = worker; item < items && ok; item += nworkers) {
    const int nxt_item = item + nworkers;
    const bool has_next = nxt_item < items;
    uint8_t *rec = cur.rec;
    // overlapped schedule: no more than `window` chunks ahead of this chain's state pass
    // (the item's first global writes, in P1, come after the barrier below)
    if (OVERLAP && p.progress && tid == 0) {
        const int need = cur.tl / C - p.window;
        if (need > 0)
            ok = progress_wait_bounded(p.progress + 2 * kProgStride * (cur.b * H + cur.h), need) && ok;
    }
    // g, k, q (tensor loads) and beta (cp.async); V may still be in flight.  One warp
    // polls the load barriers and the CTA barrier passes the loads' completion (and
    // their data) on to the rest, instead of 256 threads polling the same words.
    if (warp == 0) {
        ok = wait_ld(0) && ok;
        ok = wait_ld(1) && ok;
        ok = wait_ld(2) && ok;
    } else {
        pend &= ~7u;
    }
    cp_async_wait<0>();
    ok = cta_and(ok) != 0;
    if (!ok) break;

    // ---- P1: cumulative decay and the scaled operands ----
    // thread -> channel pair (c0, c0+1) x sub-tile a1 (rows 16a1..16a1+15).  gam holds
    // the cumsum local to the sub-tile, in log2 units; g rows past the chunk's length
    // (zeros past the tensor, or the next packed sequence's tokens) count as zero.
    const int c0 = 2 * (tid & 63), a1 = tid >> 6;
    float2 gam[ST];
    bool dense;
    {
        float2 run = make_float2(0.f, 0.f);
        const uint8_t *gsrc = (a1 < 2 ? sm.ka : sm.xk) + (a1 & 1) * ST * (D * 4) + c0 * 4;
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const float2 gv = *reinterpret_cast<const float2 *>(gsrc + j * (D * 4));
            const bool in = a1 * ST + j < cur.len;
            run.x += in ? gv.x * kLog2e : 0.f;
            run.y += in ? gv.y * kLog2e : 0.f;
            gam[j] = run;
        }
        *reinterpret_cast<float2 *>(&sm.u.p1.tot[a1][c0]) = run;
        *reinterpret_cast<float2 *>(&sm.u.p1.ref[a1][c0]) = gam[ST / 2 - 1];
        // Dense path: when every channel decays by at most 2^-(kDenseSpan / 4) over each
        // 16-token sub-tile (so by 2^-kDenseSpan over the chunk), one reference row (31,
        // the middle) keeps k e^(G_r - G_31) and k e^(G_31 - G_i) inside the bf16 range
        // for every r, i, and the key-key and query-key blocks are two whole 64 x 64
        // products on the tensor core.  Otherwise (decays near the -5 bound) the
        // 16-token sub-tile references are used.
        dense = cta_and(run.x >= -0.25f * kDenseSpan && run.y >= -0.25f * kDenseSpan) != 0;
    }
    // (the barrier above: every g value is in registers; ka and xk may be overwritten)
    // pair factors exp(G_ref(a) - G_ref(b)) <= 1 for the off-diagonal sub-tile blocks
#pragma unroll
    for (int m = 0; m < 3; ++m) {
        const int e = tid + 256 * m, pp = e >> 7, c = e & (D - 1);
        const int pa = kPairs[pp].x, pb = kPairs[pp].y;
        float d = sm.u.p1.ref[pa][c] - sm.u.p1.ref[pb][c];
        for (int a = pb; a < pa; ++a) d += sm.u.p1.tot[a][c];
        sm.mfac[pp][c] = fast_exp2(d);
    }
    {
        float2 Ba = make_float2(0.f, 0.f), GC = make_float2(0.f, 0.f);
#pragma unroll
        for (int a = 0; a < NST; ++a) {
            const float2 x = *reinterpret_cast<const float2 *>(&sm.u.p1.tot[a][c0]);
            if (a < a1) {
                Ba.x += x.x;
                Ba.y += x.y;
            }
            GC.x += x.x;
            GC.y += x.y;
        }
        const float2 Gref = gam[ST / 2 - 1], Gend = gam[ST - 1];   // local to the sub-tile
        float2 f1, f2;
        if (dense) {   // M = G_31 = the first two sub-tiles' totals
            const float2 t0 = *reinterpret_cast<const float2 *>(&sm.u.p1.tot[0][c0]);
            const float2 t1 = *reinterpret_cast<const float2 *>(&sm.u.p1.tot[1][c0]);
            const float2 M = make_float2(t0.x + t1.x, t0.y + t1.y);
            f1 = make_float2(fast_exp2(Ba.x - M.x), fast_exp2(Ba.y - M.y));                      // 2^(Ba - G_31)
            f2 = make_float2(fast_exp2(M.x - Ba.x - Gend.x), fast_exp2(M.y - Ba.y - Gend.y));   // 2^(G_31 - Ba - Gend)
        } else {
            f1 = make_float2(fast_exp2(-Gref.x), fast_exp2(-Gref.y));                   // >= 1
            f2 = make_float2(fast_exp2(Gref.x - Gend.x), fast_exp2(Gref.y - Gend.y));   // >= 1
        }
        const float2 eB = make_float2(fast_exp2(Ba.x), fast_exp2(Ba.y));                         // <= 1
        const float2 fC = make_float2(fast_exp2(GC.x - Ba.x - Gend.x), fast_exp2(GC.y - Ba.y - Gend.y));
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const int r = a1 * ST + j;
            const int off = umma_k128(C, r, c0);
            // every factor below lies in [2^-126, 2^126]: sub-tile path, [e^-80, e^40] for
            // g in (-5, 0]; dense path, within 2^kDenseSpan
            const float2 E1 = make_float2(fast_exp2(gam[j].x), fast_exp2(gam[j].y));
            const float2 E2 = make_float2(fast_exp2(Gend.x - gam[j].x), fast_exp2(Gend.y - gam[j].y));
            // raw k sits in qa and raw q in kb at the same offset; this thread reads
            // both before it overwrites them
            const float2 kf = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.qa + off));
            const float2 qf = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.kb + off));
            *reinterpret_cast<uint32_t *>(sm.ka + off) =
                pack_bf16x2(kf.x * E1.x * f1.x, kf.y * E1.y * f1.y);          // k e^(G_r - G_ref)
            *reinterpret_cast<uint32_t *>(sm.qa + off) =
                pack_bf16x2(qf.x * E1.x * f1.x, qf.y * E1.y * f1.y);          // q e^(G_r - G_ref)
            *reinterpret_cast<uint32_t *>(sm.kb + off) =
                pack_bf16x2(kf.x * E2.x * f2.x, kf.y * E2.y * f2.y);          // k e^(G_ref - G_r)
            // (G_ref: the sub-tile's reference row, or row 31 on the dense path)
            *reinterpret_cast<uint32_t *>(sm.xk + off) =
                pack_bf16x2(kf.x * E1.x * eB.x, kf.y * E1.y * eB.y);          // k e^G_r
            *reinterpret_cast<uint32_t *>(rec + REC_QG_SCRATCH + off) =
                pack_bf16x2(qf.x * E1.x * eB.x, qf.y * E1.y * eB.y);          // q e^G_r
            *reinterpret_cast<uint32_t *>(rec + REC_KT_SCRATCH + off) =
                pack_bf16x2(kf.x * E2.x * fC.x, kf.y * E2.y * fC.y);          // k e^(G_C - G_r)
        }
        if (a1 == NST - 1)
            *reinterpret_cast<float2 *>(rec + REC_GC + c0 * 4) =
                make_float2(fast_exp2(GC.x), fast_exp2(GC.y));
    }
    fence_proxy_async_smem();   // the dense path's products read ka, qa, kb
    t5::fence_before_sync();
    cta_sync();

    // ---- P2: key-key and query-key blocks ----
    // (I + A_aa)^-1 of diagonal sub-tile blocks: lane -> (block a0 + lane/16, column j)
    // (lanes 16-31 only when two blocks are given): solve (I + A_aa) x = e_j in fp32,
    // column by column (x_i is final when row i is reached; depth 16, not 120)
    auto invert_diagonal = [&](int a0) {
        const int a = a0 + (lane >> 4), j = lane & 15;
        float x[ST];
#pragma unroll
        for (int r = 0; r < ST; ++r) x[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < ST - 1; ++i)
#pragma unroll
            for (int r = i + 1; r < ST; ++r) x[r] = fmaf(-sm.u.akd[a][r][i], x[i], x[r]);
#pragma unroll
        for (int r = 0; r < ST; ++r) sm.taa[a][r * (ST + 8) + j] = f2bf(x[r]);
    };
    if (dense) {
        const uint32_t tmem = sm.tmem_slot;
        // Two tcgen05 products with the row-31 reference: A_kk = Kl Kr^T and
        // A_qk = Ql Kr^T (M = 64, N = 64, K = 128; ka, qa, kb all K-major), into tensor
        // memory columns 0-63 and 64-127; then every thread takes its rows of one block
        // (warps 0-3: A_kk, 4-7: A_qk) to the masked, beta-scaled forms the
        // substitution and the record products use.
        if (warp == 0) {
            if (t5::elect_one()) {
                t5::fence_after_sync();
                const uint64_t kd = t5::smem_desc(s_ka, 16, 1024, t5::kSwz128);
                const uint64_t qd = t5::smem_desc(s_qa, 16, 1024, t5::kSwz128);
                const uint64_t bd = t5::smem_desc(s_kb, 16, 1024, t5::kSwz128);
                constexpr uint32_t id = t5::idesc_bf16(64, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint64_t o = (uint64_t)(((ks >> 2) * C * 128 + (ks & 3) * 32) >> 4);
                    t5::mma_bf16(tmem, kd + o, bd + o, id, ks > 0);
                    t5::mma_bf16(tmem + 64, qd + o, bd + o, id, ks > 0);
                }
                t5::commit(&sm.mma_bar);
            }
            __syncwarp();
        }
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sm.mma_bar, mma_phase++ & 1));
        t5::fence_after_sync();
        if (ok) {   // M = 64 accumulators: rows 16(w&3) + gid (+8) = sub-tile w&3
            const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
            const bool kk = warp < 4;
            const int rb = (warp & 3) * 16 + gid;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float vv[16];
                t5::ld16x256b_x4(tmem + lane_base + (kk ? 0 : 64) + half * 32, vv);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = rb + 8 * hh, i = half * 32 + j8 * 8 + 2 * tig;
                        const float x0 = vv[4 * j8 + 2 * hh], x1 = vv[4 * j8 + 2 * hh + 1];
                        const int ar = r / ST, bi = i / ST;
                        if (bi > ar) continue;                       // upper blocks: unused / zero
                        if (kk) {
                            const float br = sm.beta[r];
                            if (bi < ar) {
                                *reinterpret_cast<uint32_t *>(sm.akkn + r * LDA + i) =
                                    pack_bf16x2(-x0 * br, -x1 * br);
                            } else {
                                sm.u.akd[ar][r % ST][i % ST] = (i < r) ? x0 * br : 0.f;
                                sm.u.akd[ar][r % ST][i % ST + 1] = (i + 1 < r) ? x1 * br : 0.f;
                            }
                        } else {
                            *reinterpret_cast<uint32_t *>(sm.aqk + umma_k128(C, r, i)) =
                                pack_bf16x2(i <= r ? x0 : 0.f, i + 1 <= r ? x1 : 0.f);
                        }
                    }
            }
        }
        // warps 0-3 hold their own sub-tile's diagonal block: invert it at once, while
        // warps 4-7 still write the query-key rows
        if (warp < 4) {
            __syncwarp();
            if (lane < ST) invert_diagonal(warp);
        }
        t5::fence_before_sync();
    } else {
    if (warp < 6) {
        const int a = kPairs[warp].x, b = kPairs[warp].y;
        float ak[2][4] = {}, aq[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t lk[4], lq[4], bfr[4];
            ldsm_x4(lk, s_ka + umma_k128(C, a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
            ldsm_x4(lq, s_qa + umma_k128(C, a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
            ldsm_x4(bfr, s_kb + umma_k128(C, b * ST + frag_bn_row(lane), ks * 16 + frag_bn_col(lane)));
            // right rows of sub-tile b move their reference from G_ref(b) to G_ref(a)
            const int cc = ks * 16 + 2 * tig;
            const float2 m01 = *reinterpret_cast<const float2 *>(&sm.mfac[warp][cc]);
            const float2 m89 = *reinterpret_cast<const float2 *>(&sm.mfac[warp][cc + 8]);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 x = unpack_bf16x2(bfr[u]);
                bfr[u] = (u & 1) ? pack_bf16x2(x.x * m89.x, x.y * m89.y)
                                 : pack_bf16x2(x.x * m01.x, x.y * m01.y);
            }
            mma_bf16_16816(ak[0], lk, bfr[0], bfr[1]);
            mma_bf16_16816(ak[1], lk, bfr[2], bfr[3]);
            mma_bf16_16816(aq[0], lq, bfr[0], bfr[1]);
            mma_bf16_16816(aq[1], lq, bfr[2], bfr[3]);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = a * ST + gid + 8 * hh, i = b * ST + nt * 8 + 2 * tig;
                const float br = sm.beta[r];
                *reinterpret_cast<uint32_t *>(sm.akkn + r * LDA + i) =
                    pack_bf16x2(-ak[nt][2 * hh] * br, -ak[nt][2 * hh + 1] * br);
                *reinterpret_cast<uint32_t *>(sm.aqk + umma_k128(C, r, i)) =
                    pack_bf16x2(aq[nt][2 * hh], aq[nt][2 * hh + 1]);
            }
    } else {
        const int a0 = 2 * (warp - 6);
        float aq[2][2][4] = {};
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            const int a = a0 + d;
            float ak[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t lk[4], lq[4], bfr[4];
                ldsm_x4(lk, s_ka + umma_k128(C, a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
                ldsm_x4(lq, s_qa + umma_k128(C, a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
                ldsm_x4(bfr, s_kb + umma_k128(C, a * ST + frag_bn_row(lane), ks * 16 + frag_bn_col(lane)));
                mma_bf16_16816(ak[0], lk, bfr[0], bfr[1]);
                mma_bf16_16816(ak[1], lk, bfr[2], bfr[3]);
                mma_bf16_16816(aq[d][0], lq, bfr[0], bfr[1]);
                mma_bf16_16816(aq[d][1], lq, bfr[2], bfr[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rl = gid + 8 * hh, il = nt * 8 + 2 * tig;
                    const float br = sm.beta[a * ST + rl];
                    sm.u.akd[a][rl][il] = (il < rl) ? ak[nt][2 * hh] * br : 0.f;
                    sm.u.akd[a][rl][il + 1] = (il + 1 < rl) ? ak[nt][2 * hh + 1] * br : 0.f;
                }
        }
        __syncwarp();
        invert_diagonal(a0);
#pragma unroll
        for (int d = 0; d < 2; ++d)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rl = gid + 8 * hh, il = nt * 8 + 2 * tig;
                    const int r = (a0 + d) * ST + rl, i = (a0 + d) * ST + il;
                    *reinterpret_cast<uint32_t *>(sm.aqk + umma_k128(C, r, i)) =
                        pack_bf16x2(il <= rl ? aq[d][nt][2 * hh] : 0.f,
                                    il + 1 <= rl ? aq[d][nt][2 * hh + 1] : 0.f);
                }
    }
    }
    cta_sync();

    // ---- P3: T' = (I + A)^-1 Diag(b) by blocked forward substitution, transposed ----
    // (I + A) T' = Diag(b), solved per 16-row block a:
    //   T'_a = (I + A_aa)^-1 (Diag(b)_a - sum_{c<a} A_ac T'_c).
    // Warp b (b < 4) owns columns 16b..16b+15 (above row block b, T' is zero) and works
    // with the transposes X_a = (T'_a restricted to them)^T: X_a = Z^T (I + A_aa)^-T with
    // Z^T = sum_c X_c (-A_ac)^T.  Every product's accumulator is, repacked to bf16, the
    // A operand of the next one, so the whole chain stays in registers; each X_a is
    // written to T' with transposing matrix stores.
    if (warp < NST) {
        const int b = warp;
        const uint32_t s_tp = s_ka;   // T' (umma_k128 plane, 64 x 64 bf16)
        for (int a = 0; a < b; ++a)   // row blocks above b: zero
            *reinterpret_cast<uint4 *>(sm.ka + umma_k128(C, a * ST + (lane >> 1), b * ST + 8 * (lane & 1))) =
                make_uint4(0u, 0u, 0u, 0u);
        uint32_t X[NST][4];           // bf16 A fragments of X_c, c = b .. a-1
        const int brow = (lane & 7) + 8 * (lane >> 4), bcol = 8 * ((lane >> 3) & 1);   // x4 B tiles
#pragma unroll
        for (int a = 0; a < NST; ++a) {
            if (a < b) continue;
            uint32_t za[4];
            if (a == b) {   // Z^T = Diag(b) on the block: diagonal entries only
                const float* bt = sm.beta + b * ST + 2 * tig;
                za[0] = pack_bf16x2(gid == 2 * tig ? bt[0] : 0.f, gid == 2 * tig + 1 ? bt[1] : 0.f);
                za[1] = 0u;
                za[2] = 0u;
                za[3] = pack_bf16x2(gid == 2 * tig ? bt[8] : 0.f, gid == 2 * tig + 1 ? bt[9] : 0.f);
            } else {
                float z[2][4] = {};
#pragma unroll
                for (int c = 0; c < NST; ++c) {
                    if (c < b || c >= a) continue;
                    uint32_t bf[4];   // (-A_ac)^T: akkn rows of block a, columns of block c
                    ldsm_x4(bf, smem_u32(sm.akkn + (a * ST + brow) * LDA + c * ST + bcol));
                    mma_bf16_16816(z[0], X[c], bf[0], bf[1]);
                    mma_bf16_16816(z[1], X[c], bf[2], bf[3]);
                }
                za[0] = pack_bf16x2(z[0][0], z[0][1]);
                za[1] = pack_bf16x2(z[0][2], z[0][3]);
                za[2] = pack_bf16x2(z[1][0], z[1][1]);
                za[3] = pack_bf16x2(z[1][2], z[1][3]);
            }
            uint32_t tb[4];   // (I + A_aa)^-T
            ldsm_x4(tb, smem_u32(sm.taa[a] + brow * (ST + 8) + bcol));
            float x[2][4] = {};
            mma_bf16_16816(x[0], za, tb[0], tb[1]);
            mma_bf16_16816(x[1], za, tb[2], tb[3]);
            X[a][0] = pack_bf16x2(x[0][0], x[0][1]);
            X[a][1] = pack_bf16x2(x[0][2], x[0][3]);
            X[a][2] = pack_bf16x2(x[1][0], x[1][1]);
            X[a][3] = pack_bf16x2(x[1][2], x[1][3]);
            // T' rows 16a..16a+15, columns 16b..16b+15 = X_a^T; tile m = (column half m&1,
            // row half m>>1)
            const int m = lane >> 3;
            stsm_x4_t(s_tp + umma_k128(C, a * ST + 8 * (m >> 1) + (lane & 7), b * ST + 8 * (m & 1)),
                      X[a][0], X[a][1], X[a][2], X[a][3]);
        }
    }

    const Item nxt = locate(has_next ? nxt_item : item);   // its loads start in P4

    // ---- P4: three tcgen05 products, accumulators in tensor memory (256 columns) ----
    //   Y  = T' [K*exp G | V]  (M = 64, N = 256, K = 64):  [W|U], to shared memory as bf16
    //   D1 = Kt^T [W|U]        (M = 128 key rows):         M' = -D1[:, :128], R = D1[:, 128:]
    //   D2 = Aqk  [W|U]        (M = 64 chunk rows):        Q' = Qg - D2[:, :128], O0 = D2[:, 128:]
    {
        const uint32_t tmem = sm.tmem_slot;
        if (warp == 0) ok = wait_ld(3) && ok;   // V (read by the tensor core only)
        else pend &= ~8u;
        fence_proxy_async_smem();   // T' (generic stores) -> tensor core
        t5::fence_before_sync();
        ok = cta_and(ok) != 0;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        if (ok && warp == 0) {
            if (t5::elect_one()) {
                t5::fence_after_sync();
                const uint64_t tdesc = t5::smem_desc(s_ka, 16, 1024, t5::kSwz128);                  // T', K-major
                const uint64_t xdesc = t5::smem_desc(smem_u32(sm.xk), C * 128, 1024, t5::kSwz128);  // X, N-major
                constexpr uint32_t id = t5::idesc_bf16(64, 2 * D, 0, 1);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    t5::mma_bf16(tmem, tdesc + (uint64_t)((ks * 32) >> 4),
                                 xdesc + (uint64_t)((ks * 2048) >> 4), id, ks > 0);
                t5::commit(&sm.mma_bar);
            }
            __syncwarp();
        }
        ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(&sm.mma_bar, mma_phase++ & 1));
        t5::fence_after_sync();
        // X is consumed: bring Kt (into xk) and Qg (into xv) back from the record's scratch
        // area while [W|U] leaves tensor memory; T' is consumed too: the next item's g
        // rows 0-31 go to ka
#pragma unroll
        for (int it = 0; it < 2 * C * D * 2 / 16 / 256; ++it) {
            const int i = tid + it * 256;                  // 16-byte chunk index
            const int m = i / (C * D * 2 / 16), off = (i % (C * D * 2 / 16)) * 16;
            cp_async16((m == 0 ? sm.xk : sm.xv) + off,
                       rec + (m == 0 ? REC_KT_SCRATCH : REC_QG_SCRATCH) + off);
        }
        cp_async_commit();
        if (has_next) issue(0, nxt, ld_phase + 1);
        if (ok) {   // M = 64 accumulator: rows 16(w&3)..+15; warps 0-3 -> W, warps 4-7 -> U
            const int r0 = (warp & 3) * 16 + gid, cb = (warp >> 2) * D;
#pragma unroll
            for (int qq = 0; qq < D / 32; ++qq) {
                float vv[16];
                t5::ld16x256b_x4(tmem + lane_base + cb + qq * 32, vv);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    const int c = cb + qq * 32 + j8 * 8 + 2 * tig;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        *reinterpret_cast<uint32_t *>(sm.qa + umma_k128(C, r0 + 8 * hh, c)) =
                            pack_bf16x2(vv[4 * j8 + 2 * hh], vv[4 * j8 + 2 * hh + 1]);
                }
            }
        }
        cp_async_wait<0>();         // Kt and Qg
        fence_proxy_async_smem();   // [W|U] (generic stores), Kt (cp.async) -> tensor core
        t5::fence_before_sync();
        ok = cta_and(ok) != 0;
        const uint64_t ydesc = t5::smem_desc(s_qa, C * 128, 1024, t5::kSwz128);   // [W|U], N-major
        if (ok && warp == 0) {
            if (t5::elect_one()) {
                t5::fence_after_sync();
                const uint64_t kdesc = t5::smem_desc(smem_u32(sm.xk), C * 128, 1024, t5::kSwz128);  // Kt^T, M-major
                constexpr uint32_t id = t5::idesc_bf16(128, 2 * D, 1, 1);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    t5::mma_bf16(tmem, kdesc + (uint64_t)((ks * 2048) >> 4),
                                 ydesc + (uint64_t)((ks * 2048) >> 4), id, ks > 0);
                t5::commit(&sm.mma_bar);
            }
            __syncwarp();
        }
        ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(&sm.mma_bar, mma_phase++ & 1));
        t5::fence_after_sync();
        if (has_next) issue(1, nxt, ld_phase + 1);   // Kt is consumed: g rows 32-63 to xk
        if (ok) {   // lane = key row; warps 0-3 -> M' (columns 0..127), warps 4-7 -> R
            const int m = (warp & 3) * 32 + lane, cb = (warp >> 2) * D;
#pragma unroll
            for (int qq = 0; qq < D / 32; ++qq) {
                float vv[32];
                t5::ld32(tmem + lane_base + cb + qq * 32, vv);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const int c = qq * 32 + c8 * 8;
                    const float sg = warp < 4 ? -1.f : 1.f;
                    uint4 pk;
                    pk.x = pack_bf16x2(sg * vv[c8 * 8 + 0], sg * vv[c8 * 8 + 1]);
                    pk.y = pack_bf16x2(sg * vv[c8 * 8 + 2], sg * vv[c8 * 8 + 3]);
                    pk.z = pack_bf16x2(sg * vv[c8 * 8 + 4], sg * vv[c8 * 8 + 5]);
                    pk.w = pack_bf16x2(sg * vv[c8 * 8 + 6], sg * vv[c8 * 8 + 7]);
                    uint8_t *dst = rec + (warp < 4 ? REC_M : REC_R) + core_off(D, m, c);
                    *reinterpret_cast<uint4 *>(dst) = pk;
                }
            }
        }
        t5::fence_before_sync();
        ok = cta_and(ok) != 0;
        if (ok && warp == 0) {
            if (t5::elect_one()) {
                t5::fence_after_sync();
                const uint64_t adesc = t5::smem_desc(smem_u32(sm.aqk), 16, 1024, t5::kSwz128);
                constexpr uint32_t id = t5::idesc_bf16(64, 2 * D, 0, 1);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    t5::mma_bf16(tmem, adesc + (uint64_t)((ks * 32) >> 4),
                                 ydesc + (uint64_t)((ks * 2048) >> 4), id, ks > 0);
                t5::commit(&sm.mma_bar);
            }
            __syncwarp();
        }
        ok = ok && __all_sync(0xffffffffu, mbar_wait_bounded(&sm.mma_bar, mma_phase++ & 1));
        t5::fence_after_sync();
        if (has_next) issue(2, nxt, ld_phase + 1);   // [W|U] is consumed: next k, q, beta
        if (ok) {   // M = 64 accumulator: rows 16(w&3)..+15; warps 0-3 -> Q', warps 4-7 -> O0
            const int r0 = (warp & 3) * 16 + gid, cb = (warp >> 2) * D;
            uint8_t *dst0 = rec + (warp < 4 ? REC_QP : REC_O0);
#pragma unroll
            for (int qq = 0; qq < D / 32; ++qq) {
                float vv[16];
                t5::ld16x256b_x4(tmem + lane_base + cb + qq * 32, vv);
#pragma unroll
                for (int j8 = 0; j8 < 4; ++j8) {
                    const int c = qq * 32 + j8 * 8 + 2 * tig;   // column within Q' / O0
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int r = r0 + 8 * hh;
                        float x0 = vv[4 * j8 + 2 * hh], x1 = vv[4 * j8 + 2 * hh + 1];
                        if (warp < 4) {   // Q' = Qg - Aqk W
                            const float2 f = unpack_bf16x2(
                                *reinterpret_cast<const uint32_t *>(sm.xv + umma_k128(C, r, c)));
                            x0 = f.x - x0;
                            x1 = f.y - x1;
                        }
                        *reinterpret_cast<uint32_t *>(dst0 + core_off(C, r, c)) = pack_bf16x2(x0, x1);
                    }
                }
            }
        }
        // the record's generic stores, ordered before the state pass's bulk copies of it
        if (OVERLAP) fence_proxy_async_global();
        t5::fence_before_sync();
        ok = cta_and(ok) != 0;   // Qg in xv is consumed; the record is whole
        t5::fence_after_sync();
        // publish the record (the barrier ordered every thread's stores before this
        // thread's release); not thread 0, which issues the loads: its fence would wait
        // for them
        if (OVERLAP && ok && tid == 32) {
            __threadfence();
            flag_release(p.ready + cur.idx, 1);
        }
        if (has_next) issue(3, nxt, ld_phase + 1);
    }
    cur = nxt;
    ++ld_phase;
    }   // item loop

    if (!ok && tid == 0) atomicOr(err_word, ERR_TIMEOUT_BIT);
    // nothing may land in shared memory after the CTA ends: loads still in flight (after
    // a wait that gave up) are waited for, again with the time limit
    for (int grp = 0; grp < 4; ++grp)
        if (pend & (1u << grp)) wait_ld(grp);
    cp_async_wait<0>();
}

__global__ void __launch_bounds__(kPrepThreads, 2)
kda_tc_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                   const __grid_constant__ PrepArgs p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment: the swizzled operand tiles are read by the tensor core
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(
        smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    if (threadIdx.x < 32) {   // 2D tensor-memory columns, reused by the three products
        t5::alloc(&sm.tmem_slot, 2 * D);
        t5::relinquish();
    }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    prep_worker<false>(tm_q, tm_k, tm_v, tm_g, p, sm);
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    if (threadIdx.x < 32) t5::dealloc(sm.tmem_slot, 2 * D);
}

// ---------------------------------------------------------------------------
// Kernel 2: inter-chunk state pass on tcgen05, warp-specialised.
// grid = units * tiles CTAs of 32 (NSW + 7) threads.  A unit is one (sequence,
// head) chain, or with a T-split one of its nseg consecutive segments (equal
// numbers of chunks, the last may be shorter or empty); tiles = D / DVT column
// slices of the state.  Roles:
//   NSW = 4 DVT/32 state warps: warp w's thread owns key row 32 (w % 4) + lane,
//                        columns 32 (w / 4) .. + 31 of the fp32 state tile
//                        S[:, col0:col0+DVT], in registers; per chunk it applies
//                        S <- exp(G_C) S + R + (M' S) and writes the bf16 copy of
//                        the new state that the next products read;
//   1 MMA warp:          one elected lane issues, per chunk,
//                          D_S        = M'(j) S   (M = 128 key rows, N = DVT, K = 128)
//                          D_O[j & 1] = Q'(j) S   (M = 64 chunk rows)
//                        on tcgen05, accumulating in tensor memory; D_S by 32-row K
//                        slabs as the state warps hand them over, and only then the
//                        waits for D_O's ring slot and accumulator;
//   4 output warps:      O = D_O + O0 for the chunk's rows (warp w reads tensor-memory
//                        lane quarter w % 4), stored as bf16;
//   2 producer warps:    bulk copies of the chunk records into two rings, the state
//                        ring (M', exp(G_C), R slice) and the output ring (Q', O0 slice),
//                        one warp each, refilling a slot once its consumers release it
//                        (one lane of each warp: two divergent lanes of one warp delayed
//                        the state ring's copies while the other lane spun on its wait).
// The roles hand off through mbarriers only, so the loop-carried path per chunk is
// M' S on the tensor core -> state update -> bf16 copy -> next M' S.  Every wait is
// bounded; a wait that runs out sets the shared abort flag and the timeout bit, all
// roles stop, the CTA drains what it issued, frees its tensor memory and returns.
//
// Modes.  kStateOutput: the pass proper -- outputs for every chunk, the unit's
// starting state from h0 (or s_in, per unit, after a T-split), the final state to
// hT (last segment only), and with ckpt_chunks > 0 the state after every ckpt_chunks
// whole chunks of each sequence (prefix-cache checkpoints; the segment offset keeps
// the count per sequence).  kStateMap: the first pass of the T-split -- the unit's
// affine map S_out = P S_in + R over its segment, obtained by running the same
// recurrence on a widened state [R | P] of 2D columns: the R half from zero with
// the records' R added, the P half from the identity without it (the map is affine,
// so these are its offset and its linear part).  No outputs; [R | P] goes to seg_map.
// ---------------------------------------------------------------------------
constexpr int kStateOutput = 0, kStateMap = 1;

struct StateArgs {
    const uint8_t *recs;      // chunk records
    const float *h0;          // [N, H, D, D] or null (zeros)
    float *hT;                // [N, H, D, D] or null
    __nv_bfloat16 *o;         // [tokens, H, D]
    int T, H, cps;            // dense layout: tokens per sequence, heads, chunks per sequence
    const int *hdr, *seq_off, *cu;   // packed layout (cu != null): chunk offsets per sequence
    int *err_word;
    int debug_drop_first_copy;
    int nseg;                 // segments per chain (1: no T-split)
    int mode;                 // kStateOutput or kStateMap
    const float *s_in;        // kStateOutput after a T-split: [units, D, D] starting states
    float *seg_map;           // kStateMap: [units, D, 2D] = [R | P] per unit
    // kStateOutput: state checkpoints every ckpt_chunks chunks of each sequence (0: none)
    // into ckpt[slot][H][D][D], ckpt_cap slots, each sequence's slots in token order
    float *ckpt;
    int ckpt_chunks;
    long long ckpt_cap;
    // extents for the debug bounds checks: tokens in o (all sequences) and chunk slots
    long long ntok;
    int max_chunks;
    // overlapped schedule: the prep's per-record ready flags (chunk * H + head), waited
    // for before each record is copied in; null when the records are all written
    const int *ready;
    // overlapped schedule: this CTA's count of chunks whose copies have started
    int *progress;
};
template <int DVT>
struct T5Layout {
    static_assert(DVT == 32 || DVT == 64, "column tile");
    static constexpr int R_BYTES = D * DVT * 2, O0_BYTES = C * DVT * 2;
    static constexpr int A_RAW = D * D * 2 + D * 4 + R_BYTES;            // M' | exp(G_C) | R
    static constexpr int A_BYTES = (A_RAW + 1023) / 1024 * 1024;
    static constexpr int A_GC = D * D * 2, A_R = A_GC + D * 4;
    static constexpr int B_BYTES = C * D * 2 + O0_BYTES;                 // Q' | O0
    static constexpr int B_O0 = C * D * 2;
    static constexpr int NA = DVT == 32 ? 3 : 2, NB = 3;
    static constexpr int SB_BYTES = D * DVT * 2;                         // one bf16 state copy
    static constexpr int OFF_B = NA * A_BYTES;
    static constexpr int OFF_SB = OFF_B + NB * B_BYTES;
    // barriers: full_a[NA] full_b[NB] a_free[NA] b_free[NB] done_s done_o[2] sb_full[4] do_free[2]
    static constexpr int OFF_BAR = OFF_SB + 2 * SB_BYTES;
    static constexpr int NBAR = 2 * (NA + NB) + 9;
    static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;   // tmem slot, abort flag, counters
    static constexpr int BYTES = OFF_MISC + 32 + 1024;    // + slack for 1024-byte alignment
    // Tensor memory: D_S[0] | D_O[0] | D_O[1] | D_S[1], DVT columns each.  D_S is
    // double-buffered by chunk parity: the next chunk's M'.S starts as soon as the
    // first state warp has handed over its K slab, while the other state warps may
    // still be reading this chunk's D_S.
    static constexpr uint32_t TMEM_COLS = DVT == 32 ? 128 : 256;
    KDA_DEVINL static uint32_t ds_col(int parity) { return parity ? 3 * DVT : 0; }
    // B operand (the state copy), MN-major: row k (key) holds DVT bf16 values.
    // DVT = 64: 128-byte rows, 128-byte swizzle; DVT = 32: 64-byte rows, 64-byte swizzle.
    static constexpr uint32_t SB_ROW = DVT * 2;
    static constexpr uint32_t SB_SWZ = DVT == 64 ? t5::kSwz128 : t5::kSwz64;
    KDA_DEVINL static int sb_off(int k, int n) {
        const int chunk = (n >> 3) ^ (DVT == 64 ? (k & 7) : ((k >> 1) & 3));
        return k * SB_ROW + (chunk << 4) + ((n & 7) << 1);
    }
    static_assert(BYTES <= 232448, "shared memory budget");
};

// Warp roles of the state pass: NSW = 4 DVT/32 state warps (warp w: key row
// 32 (w % 4) + lane, columns 32 (w / 4) .. + 31 of the slice), then the MMA warp, four
// output warps and the producer warps of the state ring and the output ring; in the
// overlapped schedule one more warp polls the records' ready flags.
template <int DVT>
struct StateRoles {
    static constexpr int NSW = 4 * (DVT / 32);
    static constexpr int MMA_WARP = NSW, OUT_WARP0 = NSW + 1, PROD_WARP = NSW + 5,
                         PROD_B_WARP = NSW + 6, POLL_WARP = NSW + 7;
    static constexpr int THREADS = 32 * (NSW + 7);
};

// One state-pass CTA: `cta` indexes (unit, column tile), column tile fastest.  Warps
// past the roles (when the block is larger) only take part in the CTA barriers.
// OVERLAP: the poller warp, the wait for published records and the progress counter
// of the overlapped schedule (compiled out of the standalone kernel: their mere
// presence in the producer's loop cost it 13% in time).
template <int DVT, bool OVERLAP>
KDA_DEVINL void state_cta(const StateArgs &a, const int cta) {
    using L = T5Layout<DVT>;
    using RL = StateRoles<DVT>;
    const uint8_t *__restrict__ recs = a.recs;
    __nv_bfloat16 *__restrict__ o = a.o;
    const int H = a.H;
    const bool map_mode = a.mode == kStateMap;
    constexpr int NA = L::NA, NB = L::NB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full_a = reinterpret_cast<uint64_t *>(sm + L::OFF_BAR);
    uint64_t *full_b = full_a + NA;
    uint64_t *a_free = full_b + NB;
    uint64_t *b_free = a_free + NA;
    uint64_t *done_s = b_free + NB;
    uint64_t *done_o = done_s + 1;     // [2] by chunk parity
    uint64_t *sb_full = done_o + 2;    // [4]: key rows 32w..32w+31 of the state copy written
    uint64_t *do_free = sb_full + 4;   // [2] by chunk parity
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + L::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 4);
    int *cnt = reinterpret_cast<int *>(sm + L::OFF_MISC + 8);   // [0] ring A issued, [1] ring B issued, [2] MMA issued
    // overlapped schedule: records known to be published, [0, *rdy) (the poller warp's count)
    volatile int *rdy = reinterpret_cast<volatile int *>(sm + L::OFF_MISC + 20);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // 1-D grid, column tile fastest so the tiles of one unit run side by side
    // and share the chunk records through L2.
    const int tiles = (map_mode ? 2 * D : D) / DVT;
    const int tile = cta % tiles, unit = cta / tiles;
    const int chain = unit / a.nseg, seg = unit % a.nseg, n = chain / H, h = chain % H;
    const bool p_half = map_mode && tile >= D / DVT;   // linear part of the map: no R
    const int col0 = (tile % (D / DVT)) * DVT;

    int c_begin, c_end, seq_t0, seq_len;
    if (a.cu) {
        if (!a.hdr[0]) return;
        c_begin = a.seq_off[n];
        c_end = a.seq_off[n + 1];
        seq_t0 = a.cu[n];
        seq_len = a.cu[n + 1] - a.cu[n];
    } else {
        c_begin = n * a.cps;
        c_end = c_begin + a.cps;
        seq_t0 = n * a.T;
        seq_len = a.T;
    }
    if constexpr (KDA_DEBUG) {   // the chain's chunks and tokens inside their buffers
        const bool bad = c_begin < 0 || c_end > a.max_chunks || c_end - c_begin != (seq_len + C - 1) / C ||
                         seq_len < 0 || seq_t0 < 0 || (long long)seq_t0 + seq_len > a.ntok;
        if (bad) {
            if (threadIdx.x == 0) atomicOr(a.err_word, ERR_BOUNDS_BIT);
            return;
        }
    }
    const int seq_tokens = seq_len;   // the whole sequence
    int seg_lo;                       // chunks of the sequence before this unit's segment
    {   // this unit's segment of the chain
        const int nch = c_end - c_begin, per = (nch + a.nseg - 1) / a.nseg;
        const int lo = min(nch, seg * per), hi = min(nch, lo + per);
        seg_lo = lo;
        c_begin += lo;
        c_end = c_begin + (hi - lo);
        seq_t0 += lo * C;
        seq_len -= lo * C;
    }
    const int nchunks = c_end - c_begin;
    int *err_word = a.err_word;

    if (tid == 0) {
        // consumers release and hand over once per warp (lane 0, after __syncwarp)
        for (int s = 0; s < NA; ++s) { mbar_init(&full_a[s], 1); mbar_init(&a_free[s], RL::NSW); }
        for (int s = 0; s < NB; ++s) { mbar_init(&full_b[s], 1); mbar_init(&b_free[s], 4); }
        mbar_init(done_s, 1);
        mbar_init(&done_o[0], 1);
        mbar_init(&done_o[1], 1);
        for (int w = 0; w < 4; ++w) mbar_init(&sb_full[w], DVT / 32);
        mbar_init(&do_free[0], 4);
        mbar_init(&do_free[1], 4);
        *abort_flag = 0;
        cnt[0] = cnt[1] = cnt[2] = 0;
        *rdy = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        t5::alloc(tmem_slot, L::TMEM_COLS);
        t5::relinquish();
    }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t sm_addr = smem_u32(sm);
    auto fail = [&]() {
        if (*abort_flag == 0) {
            *abort_flag = 1;
            atomicOr(err_word, ERR_TIMEOUT_BIT);
        }
    };
    auto rec_of = [&](int j) { return recs + ((size_t)(c_begin + j) * H + h) * REC_BYTES; };

    if (warp < RL::NSW) {
        // ---------------- state warps ----------------
        const int row = (warp & 3) * 32 + lane, cb = (warp >> 2) * 32;   // key row, columns cb..cb+31
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float S[32];
        const size_t row_off = (size_t)row * D + col0 + cb;
        const float *init = nullptr;
        if (!map_mode)
            init = a.s_in ? a.s_in + (size_t)unit * D * D + row_off
                          : (a.h0 ? a.h0 + (size_t)chain * D * D + row_off : nullptr);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (init) x = *reinterpret_cast<const float4 *>(init + i);
            S[i] = x.x;
            S[i + 1] = x.y;
            S[i + 2] = x.z;
            S[i + 3] = x.w;
        }
        if (p_half) {   // identity columns col0 + cb ..
#pragma unroll
            for (int i = 0; i < 32; ++i) S[i] = (row == col0 + cb + i) ? 1.f : 0.f;
        }
        // state checkpoints: the first slot of this sequence (its earlier sequences'
        // checkpoint counts, summed by the warp for packed input)
        const bool ckpt_on = !map_mode && a.ckpt_chunks > 0;
        long long ck_first = 0;
        if (ckpt_on) {
            const int every = a.ckpt_chunks * C;
            if (a.cu) {
                long long part = 0;
                for (int m = lane; m < n; m += 32) part += (a.cu[m + 1] - a.cu[m]) / every;
#pragma unroll
                for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                ck_first = part;
            } else {
                ck_first = (long long)n * (seq_tokens / every);
            }
        }
        auto write_sb = [&](int buf) {   // bf16 copy of this thread's part of its row, then signal
            uint8_t *sb = sm + L::OFF_SB + buf * L::SB_BYTES;
#pragma unroll
            for (int c8 = 0; c8 < 32; c8 += 8) {
                uint4 pk;
                pk.x = pack_bf16x2(S[c8], S[c8 + 1]);
                pk.y = pack_bf16x2(S[c8 + 2], S[c8 + 3]);
                pk.z = pack_bf16x2(S[c8 + 4], S[c8 + 5]);
                pk.w = pack_bf16x2(S[c8 + 6], S[c8 + 7]);
                *reinterpret_cast<uint4 *>(sb + L::sb_off(row, cb + c8)) = pk;
            }
            fence_proxy_async_smem();   // generic writes -> tensor-core reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb_full[warp & 3]);   // key rows 32(w%4).. : K slab w%4 of the next products
        };
        write_sb(0);
        int j = 0;
        for (; j < nchunks && !*abort_flag; ++j) {
            const int sa = j % NA;
            const uint8_t *st = sm + sa * L::A_BYTES;
            bool ok = mbar_wait_bounded(&full_a[sa], (j / NA) & 1);
            const float gam = reinterpret_cast<const float *>(st + L::A_GC)[row];
            uint4 rv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)   // this thread's part of R row `row` (zero for P)
                rv[i] = p_half ? make_uint4(0u, 0u, 0u, 0u)
                               : *reinterpret_cast<const uint4 *>(st + L::A_R + core_off(D, row, cb + 8 * i));
            // the tensor-memory load below is warp-collective: decide as a warp
            ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(done_s, j & 1));
            if (!ok) { fail(); break; }
            t5::fence_after_sync();
            float v[32];
            t5::ld32(tmem + lane_base + L::ds_col(j & 1) + cb, v);
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_free[sa]);   // the warp is done with the slot and with D_S
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t u[4] = {rv[i].x, rv[i].y, rv[i].z, rv[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 r2 = unpack_bf16x2(u[e]);
                    const int c = i * 8 + 2 * e;
                    S[c] = fmaf(gam, S[c], r2.x + v[c]);
                    S[c + 1] = fmaf(gam, S[c + 1], r2.y + v[c + 1]);
                }
            }
            if (j + 1 < nchunks) write_sb((j + 1) & 1);
            // after the hand-off: its arrive releases this thread's earlier stores too, so
            // checkpoint stores issued before it would hold up the next chunk's product
            if (ckpt_on) {   // S holds the state after `done` whole chunks of the sequence
                const int done = seg_lo + j + 1;
                if (done % a.ckpt_chunks == 0 && done * C <= seq_tokens) {
                    const long long slot = ck_first + done / a.ckpt_chunks - 1;
                    if (slot < a.ckpt_cap) {
                        float *cp = a.ckpt + ((slot * H + h) * D + row) * D + col0 + cb;
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(cp + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
                    } else if (lane == 0) {
                        atomicOr(err_word, ERR_CKPT_BIT);
                    }
                }
            }
        }
        float *dst = nullptr;
        if (map_mode)
            dst = a.seg_map + ((size_t)unit * D + row) * (2 * D) + tile * DVT + cb;
        else if (a.hT && seg == a.nseg - 1)
            dst = a.hT + (size_t)chain * D * D + row_off;
        if (!*abort_flag && dst && j == nchunks) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
        }
    } else if (warp == RL::MMA_WARP) {
        // ---------------- MMA warp ----------------
        constexpr uint32_t idS = t5::idesc_bf16(128, DVT, 0, 1);
        constexpr uint32_t idO = t5::idesc_bf16(64, DVT, 0, 1);
        // One lane issues every product, so each commit also covers the products it
        // issued before: done_s(j) implies the previous chunk's Q'.S is complete too.
        const bool leader = t5::elect_one();
        for (int j = 0; j < nchunks && !*abort_flag; ++j) {
            const int sa = j % NA, sbb = j % NB;
            // M'.S waits only for its ring slot and the state copy; the output product's
            // ring slot and accumulator are waited for after it is on its way
            bool ok = mbar_wait_bounded(&full_a[sa], (j / NA) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) { fail(); break; }
            bool slab_ok = true;
            const uint32_t sb_addr = sm_addr + L::OFF_SB + (j & 1) * L::SB_BYTES;
            const uint64_t bd0 = t5::smem_desc(sb_addr, 4096, 8 * L::SB_ROW, L::SB_SWZ);
            if (leader) {
                // A operands in the core-matrix layout: 8-row groups 128 B apart (SBO),
                // 8-column chunks rows*16 B apart (LBO), no swizzle.
                const uint64_t am0 = t5::smem_desc(sm_addr + sa * L::A_BYTES, D * 16, 128, 0);
                // M'.S by K slabs: slab w (key rows 32w..32w+31, two K=16 steps) goes as
                // soon as state warp w has written its rows of the copy
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (!mbar_wait_bounded(&sb_full[w], j & 1)) {
                        slab_ok = false;
                        break;
                    }
                    t5::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const int ks = 2 * w + kk;
                        t5::mma_bf16(tmem + L::ds_col(j & 1), am0 + (uint64_t)((ks * 2 * D * 16) >> 4),
                                     bd0 + (uint64_t)((ks * 16 * L::SB_ROW) >> 4), idS, ks > 0);
                    }
                }
                t5::commit(done_s);
            }
            bool ok2 = !__any_sync(0xffffffffu, !slab_ok);
            ok2 = ok2 && (map_mode || (mbar_wait_bounded(&full_b[sbb], (j / NB) & 1) &&
                                       (j < 2 || mbar_wait_bounded(&do_free[j & 1], ((j - 2) >> 1) & 1))));
            ok2 = __all_sync(0xffffffffu, ok2);
            if (leader) {
                if (!map_mode) {
                    if (ok2) {
                        const uint64_t aq0 = t5::smem_desc(sm_addr + L::OFF_B + sbb * L::B_BYTES,
                                                           C * 16, 128, 0);
                        const uint32_t dO = tmem + DVT + (j & 1) * DVT;
                        t5::fence_after_sync();
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks)
                            t5::mma_bf16(dO, aq0 + (uint64_t)((ks * 2 * C * 16) >> 4),
                                         bd0 + (uint64_t)((ks * 16 * L::SB_ROW) >> 4), idO, ks > 0);
                    }
                    t5::commit(&done_o[j & 1]);   // always: the drain below waits on it
                }
                cnt[2] = j + 1;
            }
            if (!ok2) { fail(); break; }
        }
    } else if (warp < RL::PROD_WARP) {
        // ---------------- output warps (none in the map pass) ----------------
        const int q = warp & 3;                          // tensor-memory lane quarter
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int orow = q * 16 + lane;                  // output row of lanes 0..15
        for (int j = 0; j < (map_mode ? 0 : nchunks) && !*abort_flag; ++j) {
            const int sbb = j % NB;
            bool ok = mbar_wait_bounded(&done_o[j & 1], (j >> 1) & 1) &&
                      mbar_wait_bounded(&full_b[sbb], (j / NB) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) { fail(); break; }
            t5::fence_after_sync();
            float w[DVT];
            t5::ld_cols<DVT>(tmem + lane_base + DVT + (j & 1) * DVT, w);
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&do_free[j & 1]);
            const int t0 = seq_t0 + j * C;
            const int len = min(C, seq_len - j * C);
            if (lane < 16 && orow < len) {
                const uint8_t *op0 = sm + L::OFF_B + sbb * L::B_BYTES + L::B_O0;
                __nv_bfloat16 *op = o + ((size_t)(t0 + orow) * H + h) * D + col0;
#pragma unroll
                for (int i = 0; i < DVT / 8; ++i) {
                    const uint4 ov = *reinterpret_cast<const uint4 *>(op0 + core_off(C, orow, 8 * i));
                    const uint32_t u[4] = {ov.x, ov.y, ov.z, ov.w};
                    uint4 res;
                    uint32_t *rr = reinterpret_cast<uint32_t *>(&res);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 o2 = unpack_bf16x2(u[e]);
                        rr[e] = pack_bf16x2(w[i * 8 + 2 * e] + o2.x, w[i * 8 + 2 * e + 1] + o2.y);
                    }
                    *reinterpret_cast<uint4 *>(op + i * 8) = res;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_free[sbb]);
        }
    } else if (OVERLAP && warp == RL::POLL_WARP) {
        // ---------------- poller (overlapped schedule only; the fused block's spare warp) ----------------
        // walks the chain's records in order, waiting (acquire, GPU scope) for each ready
        // flag the prep sets, and counts the published ones in shared memory, so the
        // producer's copies never wait on a global-memory round trip
        if (lane == 0) {
            for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                if (!flag_wait_bounded(a.ready + (size_t)(c_begin + c) * H + h)) { fail(); break; }
                __threadfence_block();   // the acquired state first, then the count (CTA scope)
                *rdy = c + 1;
            }
        }
        __syncwarp();
    } else if (warp == RL::PROD_WARP || warp == RL::PROD_B_WARP) {
        // ---------------- producer warps: lane 0 of each feeds ring A, ring B ----------------
        // overlapped schedule: a record is copied in only once the poller has seen it published
        auto ready = [&](int c) {
            if constexpr (!OVERLAP) return true;
            if (*rdy <= c) {
                const uint64_t t0 = global_timer_ns();
                while (*rdy <= c) {
                    if (*abort_flag || global_timer_ns() - t0 > kWaitLimitNs) return false;
                }
            }
            __threadfence_block();
            fence_proxy_async_global();   // the prep's generic stores -> these bulk copies
            return true;
        };
        if (lane == 0 && warp == RL::PROD_WARP) {
            for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                const int s = c % NA;
                if (c >= NA && !mbar_wait_bounded(&a_free[s], ((c - NA) / NA) & 1)) { fail(); break; }
                if (!ready(c)) { fail(); break; }
                fence_proxy_async_smem();
                uint64_t *bar = &full_a[s];
                uint8_t *dst = sm + s * L::A_BYTES;
                const uint8_t *rec = rec_of(c);
                mbar_arrive_expect_tx(bar, p_half ? L::A_RAW - L::R_BYTES : L::A_RAW);
                cnt[0] = c + 1;
                if (a.debug_drop_first_copy && c == 0) continue;   // test hook: the wait must run out
                bulk_g2s(dst, rec + REC_M, D * D * 2, bar);
                bulk_g2s(dst + L::A_GC, rec + REC_GC, D * 4, bar);
                if (!p_half)
                    bulk_g2s(dst + L::A_R, rec + REC_R + core_off(D, 0, col0), L::R_BYTES, bar);
                // a hint for the prep's throttle: a relaxed store, no fence (a release
                // here would hold this lane until its earlier copies are done)
                if constexpr (OVERLAP) store_relaxed(a.progress + kProgStride * cta, c + 1);
            }
        } else if (lane == 0) {
            for (int c = 0; c < (map_mode ? 0 : nchunks) && !*abort_flag; ++c) {
                const int s = c % NB;
                if (c >= NB && !mbar_wait_bounded(&b_free[s], ((c - NB) / NB) & 1)) { fail(); break; }
                if (!ready(c)) { fail(); break; }
                fence_proxy_async_smem();
                uint64_t *bar = &full_b[s];
                uint8_t *dst = sm + L::OFF_B + s * L::B_BYTES;
                const uint8_t *rec = rec_of(c);
                mbar_arrive_expect_tx(bar, L::B_BYTES);
                cnt[1] = c + 1;
                bulk_g2s(dst, rec + REC_QP, C * D * 2, bar);
                bulk_g2s(dst + L::B_O0, rec + REC_O0 + core_off(C, 0, col0), L::O0_BYTES, bar);
            }
        }
        __syncwarp();
    }

    t5::fence_before_sync();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let what this CTA issued finish (bounded) before its shared memory goes
        for (int c = max(0, cnt[0] - NA); c < cnt[0]; ++c)
            mbar_wait_bounded(&full_a[c % NA], (c / NA) & 1);
        for (int c = max(0, cnt[1] - NB); c < cnt[1]; ++c)
            mbar_wait_bounded(&full_b[c % NB], (c / NB) & 1);
        if (map_mode) {   // done_s is the last commit of each chunk
            if (cnt[2] > 0) mbar_wait_bounded(done_s, (cnt[2] - 1) & 1);
        } else {
            for (int c = max(0, cnt[2] - 2); c < cnt[2]; ++c)
                mbar_wait_bounded(&done_o[c & 1], (c >> 1) & 1);
        }
    }
    __syncthreads();
    t5::fence_after_sync();
    if (warp == 0) t5::dealloc(tmem, L::TMEM_COLS);
}

template <int DVT>
__global__ void __launch_bounds__(StateRoles<DVT>::THREADS, 1) kda_tc_state_kernel(const __grid_constant__ StateArgs a) {
    state_cta<DVT, false>(a, blockIdx.x);
}

// ---------------------------------------------------------------------------
// Overlapped schedule: kernels 1 and 2 as one launch (fixed-length input).
// The first `nstate` CTAs run the state pass on 64-column slices (one per SM), the
// others each run two prep workers (the two CTAs of kernel 1's usual two per SM, as
// one block, with their own shared memory, tensor-memory columns and named barriers)
// over the records in time order.  A state CTA waits for a record's ready flag
// before copying it in, so the state chain starts after the first records instead
// of after all of them, and the prep runs on the SMs the chain leaves idle; a prep
// worker stays within a window of chunks ahead of its chain's state CTAs.  Every
// wait is for work earlier in time order than what the waiter holds (no cycle) and
// bounded, and the grid is one block per SM, launched cooperatively so all blocks
// are resident.
// ---------------------------------------------------------------------------
constexpr int kFusedThreads = 2 * kPrepThreads;
constexpr int kFusedPrepStride = (int)((sizeof(PrepSmem) + 1023) / 1024 * 1024);
constexpr int kFusedSmem = (2 * kFusedPrepStride + 1024 > T5Layout<64>::BYTES)
                               ? 2 * kFusedPrepStride + 1024 : T5Layout<64>::BYTES;
// the state roles and the ready-flag poller (one more warp) fit the fused block
static_assert(StateRoles<64>::THREADS + 32 <= kFusedThreads, "state roles fit the fused block");
static_assert(kFusedSmem <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kFusedThreads, 1)
kda_tc_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ PrepArgs p, const __grid_constant__ StateArgs a,
                    const int nstate) {
    if ((int)blockIdx.x < nstate) {
        state_cta<64, true>(a, blockIdx.x);
        return;
    }
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    PrepSmem &s0 = *reinterpret_cast<PrepSmem *>(base);
    const int w = threadIdx.x / kPrepThreads;
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(base + w * kFusedPrepStride);
    if (threadIdx.x < 32) {   // both workers' columns at once: one allocation per CTA
        t5::alloc(&s0.tmem_slot, 4 * D);
        t5::relinquish();
    }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    // worker 1's columns follow worker 0's; each worker reads its own slot
    if (w == 1 && threadIdx.x == kPrepThreads) sm.tmem_slot = s0.tmem_slot + 2 * D;
    __syncthreads();
    prep_worker<true>(tm_q, tm_k, tm_v, tm_g, p, sm);
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    if (threadIdx.x < 32) t5::dealloc(s0.tmem_slot, 4 * D);
}

// ---------------------------------------------------------------------------
// Kernel 3 (T-split only): the segment combine.  Walks each chain's segments in
// order, S_{s+1} = P_s S_s + R_s in fp32, and stores every segment's starting state
// S_s (S_0 = h0 or zero) for the output pass.  grid = (N * H, D / 32): one CTA per
// chain and 32-column slice of the state (columns are independent); 256 threads,
// thread t owns row t / 2, columns 16 (t & 1) .. +15 of the slice.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kda_tc_seg_combine_kernel(
    const float *__restrict__ h0, const float *__restrict__ seg_map, float *__restrict__ s_in,
    int nseg, const int *__restrict__ hdr, int packed) {
    __shared__ __align__(16) float Ssm[D][32];
    if (packed && !hdr[0]) return;
    const int chain = blockIdx.x, c0 = blockIdx.y * 32;
    const int r = threadIdx.x >> 1, cl = (threadIdx.x & 1) * 16;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h0) v = *reinterpret_cast<const float4 *>(h0 + ((size_t)chain * D + r) * D + c0 + cl + i);
        x[i] = v.x;
        x[i + 1] = v.y;
        x[i + 2] = v.z;
        x[i + 3] = v.w;
    }
    for (int s = 0; s < nseg; ++s) {
        const size_t unit = (size_t)chain * nseg + s;
        float *dst = s_in + (unit * D + r) * D + c0 + cl;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4 *>(dst + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        if (s == nseg - 1) break;
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4 *>(&Ssm[r][cl + i]) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        __syncthreads();
        const float *row = seg_map + (unit * D + r) * (2 * D);   // [R | P] row r
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(row + c0 + cl + i);
            x[i] = v.x;
            x[i + 1] = v.y;
            x[i + 2] = v.z;
            x[i + 3] = v.w;
        }
        for (int k4 = 0; k4 < D; k4 += 4) {
            const float4 p = *reinterpret_cast<const float4 *>(row + D + k4);
            const float pk[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    const float4 sv = *reinterpret_cast<const float4 *>(&Ssm[k4 + u][cl + i]);
                    x[i] = fmaf(pk[u], sv.x, x[i]);
                    x[i + 1] = fmaf(pk[u], sv.y, x[i + 1]);
                    x[i + 2] = fmaf(pk[u], sv.z, x[i + 2]);
                    x[i + 3] = fmaf(pk[u], sv.w, x[i + 3]);
                }
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Context parallelism across devices: the starting state of rank `rank`'s time
// segment.  maps holds every rank's segment map [R | P] ([world][chains][D][2D], the
// map pass's layout), gathered from all ranks; S_in(rank) = fold over ranks
// 0 .. rank-1 of S <- P_s S + R_s, from h0 (or zero).  grid = (chains, D / 32), 256
// threads: thread t owns row t / 2, columns 16 (t & 1) .. +15 of the 32-column slice.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kda_cp_combine_kernel(
    const float *__restrict__ h0, const float *__restrict__ maps, float *__restrict__ s_in,
    int rank, int chains) {
    __shared__ __align__(16) float Ssm[D][32];
    const int chain = blockIdx.x, c0 = blockIdx.y * 32;
    const int r = threadIdx.x >> 1, cl = (threadIdx.x & 1) * 16;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h0) v = *reinterpret_cast<const float4 *>(h0 + ((size_t)chain * D + r) * D + c0 + cl + i);
        x[i] = v.x;
        x[i + 1] = v.y;
        x[i + 2] = v.z;
        x[i + 3] = v.w;
    }
    for (int s = 0; s < rank; ++s) {
#pragma unroll
        for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4 *>(&Ssm[r][cl + i]) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        __syncthreads();
        const float *row = maps + (((size_t)s * chains + chain) * D + r) * (2 * D);   // [R | P]
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(row + c0 + cl + i);
            x[i] = v.x;
            x[i + 1] = v.y;
            x[i + 2] = v.z;
            x[i + 3] = v.w;
        }
        for (int k4 = 0; k4 < D; k4 += 4) {
            const float4 p = *reinterpret_cast<const float4 *>(row + D + k4);
            const float pk[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    const float4 sv = *reinterpret_cast<const float4 *>(&Ssm[k4 + u][cl + i]);
                    x[i] = fmaf(pk[u], sv.x, x[i]);
                    x[i + 1] = fmaf(pk[u], sv.y, x[i + 1]);
                    x[i + 2] = fmaf(pk[u], sv.z, x[i + 2]);
                    x[i + 3] = fmaf(pk[u], sv.w, x[i + 3]);
                }
            }
        }
        __syncthreads();
    }
    float *dst = s_in + ((size_t)chain * D + r) * D + c0 + cl;
#pragma unroll
    for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
}

}  // namespace tc
}  // namespace kda
