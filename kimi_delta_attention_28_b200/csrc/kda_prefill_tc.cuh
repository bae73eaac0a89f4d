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
// Kernel 1 (kda_tc_prep_kernel) computes every chunk-local quantity, fully in
// parallel over (chunk, head): the log-decay cumsum; the key-key and query-key
// blocks with the pairwise decays factored through 16-token sub-tile reference
// rows so no factor overflows (the same page's panel "g ∈ (-5, 0)" bounds a
// 16-token decay by e^-80); [W|U] by blocked forward substitution (fp32 inverses
// of the 16x16 diagonal blocks, tensor-core products elsewhere); the decayed keys
// and queries.  It writes one record per (chunk, head).  Kernel 2
// (kda_tc_state_kernel) walks the chunks of each (sequence, head) in order with
// the fp32 state on chip, split over d_v column tiles (state columns evolve
// independently); records arrive by bulk copies into a 3-stage ring.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace tc {

constexpr int D = 128;          // head size (d_k = d_v)
constexpr int C = 64;           // chunk length
constexpr int ST = 16;          // sub-tile length for the decay reference rows
constexpr int NST = C / ST;     // sub-tiles per chunk
constexpr int LD = D + 8;       // padded bf16 row stride of staged inputs (272 B)
constexpr int LDY = 2 * D + 8;  // padded bf16 row stride of the [W|U] solution (528 B)
constexpr int LDA = C + 8;      // padded bf16 row stride of the key-key block (144 B)

// Per (chunk, head) record, written by kernel 1 and read by kernel 2.  The
// [C][D] tiles use the swz128 layout (16-byte chunks XOR-permuted by row) so a
// plain bulk copy lands them in shared memory ready for conflict-free ldmatrix.
constexpr int REC_W = 0;                    // W                 [C][D] bf16, swz128
constexpr int REC_KT = REC_W + C * D * 2;   // K*exp(G_C - G)    [C][D] bf16, swz128
constexpr int REC_QG = REC_KT + C * D * 2;  // Q*exp(G)          [C][D] bf16, swz128
constexpr int REC_AQK = REC_QG + C * D * 2; // masked query-key  [C][C] bf16, swz64
constexpr int REC_GC = REC_AQK + C * C * 2; // exp(G_C)          [D] fp32
constexpr int REC_SHARED = REC_GC + D * 4;  // bytes every column tile reads (57,856)
constexpr int REC_U = REC_SHARED;           // U as 8 column tiles [8][C][16] bf16
constexpr int UT = 16;                      // U tile width
constexpr int REC_BYTES = REC_U + C * D * 2;  // 74,240
static_assert(REC_BYTES % 256 == 0 && REC_SHARED % 16 == 0, "record alignment");

KDA_DEVINL int rec_u_off(int r, int c) {
    return REC_U + (c >> 4) * (C * UT * 2) + r * (UT * 2) + (c & 15) * 2;
}

struct ChunkLoc {
    int t0;    // first token (flattened over the batch / packed sequences)
    int len;   // tokens in this chunk, 1..C
};

constexpr int ERR_TIMEOUT_BIT = 2;

// ---------------------------------------------------------------------------
// Varlen chunk map: validates cu_seqlens and lays out each sequence's chunks.
// One block.  hdr[0] = 1 when valid; seq_off[n] = first chunk of sequence n.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) kda_chunk_map_kernel(const int *__restrict__ cu, int N,
                                                             int T, int *hdr, int *seq_off,
                                                             ChunkLoc *chunks, int *err_word,
                                                             int err_code) {
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
// Kernel 1: intra-chunk transform.  grid = (chunk slots, H), 256 threads.
// ---------------------------------------------------------------------------
struct PrepSmem {
    // kL/qL: raw k/q, then scaled left operands; afterwards the [W|U] solution
    // (64 x LDY bf16 = 33,792 B spans both arrays, which are adjacent).
    __nv_bfloat16 kL[C * LD];      // k * exp(G_r - G_ref(a))
    __nv_bfloat16 qL[C * LD];      // q * exp(G_r - G_ref(a))
    __nv_bfloat16 v[C * LD];       // raw v
    __nv_bfloat16 kR[C * LD];      // k * exp(G_ref(b) - G_i); afterwards per-warp scratch
    __nv_bfloat16 kG[C * LD];      // k * exp(G_r)
    __nv_bfloat16 akkn[C * LDA];   // -b_r A_ri for sub-tile blocks b < a (bf16)
    float akd[NST][ST][ST + 1];    //  b_r A_ri inside diagonal sub-tile blocks (fp32)
    __nv_bfloat16 taa[NST][ST * (ST + 8)];  // (I + A_aa)^-1, bf16
    float gref[NST][D];            // G at each sub-tile's reference row (log2 units)
    float xch[NST][D];             // sub-tile decay totals
    float beta[C];
};
static_assert(sizeof(__nv_bfloat16) * C * LDY <= 2 * sizeof(__nv_bfloat16) * C * LD, "Y fits");

__global__ void __launch_bounds__(256, 2)
kda_tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, int T, int H, int cps,
                   const int *__restrict__ hdr, const ChunkLoc *__restrict__ chunks,
                   uint8_t *__restrict__ recs) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int cid = blockIdx.x, h = blockIdx.y;

    int t0, len;
    if (chunks) {
        if (!hdr[0] || cid >= hdr[1]) return;
        t0 = chunks[cid].t0;
        len = chunks[cid].len;
    } else {
        const int n = cid / cps, j = cid % cps;
        t0 = n * T + j * C;
        len = min(C, T - j * C);
    }
    uint8_t *rec = recs + ((size_t)cid * H + h) * REC_BYTES;
    const size_t rowstride = (size_t)H * D;  // elements between consecutive tokens
    const size_t base = ((size_t)t0 * H + h) * D;

    // ---- P0: stage k, q, v rows (zero-filled past len) and beta ----
#pragma unroll
    for (int it = 0; it < 3 * C * (D / 8) / 256; ++it) {
        const int i = tid + it * 256;
        const int m = i / (C * (D / 8));
        const int rem = i % (C * (D / 8));
        const int r = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
        const __nv_bfloat16 *src = (m == 0 ? k : (m == 1 ? q : v));
        __nv_bfloat16 *dst = (m == 0 ? sm.kL : (m == 1 ? sm.qL : sm.v)) + r * LD + c8;
        const bool ok = r < len;
        cp_async16(dst, ok ? (src + base + r * rowstride + c8) : src, ok ? 16 : 0);
    }
    cp_async_commit();
    if (tid < C) sm.beta[tid] = tid < len ? beta[(size_t)(t0 + tid) * H + h] : 0.f;

    // ---- P1: cumulative decay and the scaled operands ----
    // thread -> channel pair (2cp, 2cp+1) x sub-tile a (rows 16a..16a+15); log2 units.
    const int cp = tid & 63, a1 = tid >> 6, c0 = 2 * cp;
    float2 gam[ST];
    {
        float2 run = make_float2(0.f, 0.f);
        const float *gp = g + base + c0;
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const int r = a1 * ST + j;
            const float2 gv = r < len ? *reinterpret_cast<const float2 *>(gp + r * rowstride)
                                      : make_float2(0.f, 0.f);
            run.x += gv.x * kLog2e;
            run.y += gv.y * kLog2e;
            gam[j] = run;
        }
        *reinterpret_cast<float2 *>(&sm.xch[a1][c0]) = run;
    }
    cp_async_wait<0>();
    __syncthreads();
    {
        float2 Ba = make_float2(0.f, 0.f), GC = make_float2(0.f, 0.f);
#pragma unroll
        for (int a = 0; a < NST; ++a) {
            const float2 x = *reinterpret_cast<const float2 *>(&sm.xch[a][c0]);
            if (a < a1) {
                Ba.x += x.x;
                Ba.y += x.y;
            }
            GC.x += x.x;
            GC.y += x.y;
        }
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            gam[j].x += Ba.x;
            gam[j].y += Ba.y;
        }
        const float2 Gref = gam[ST / 2 - 1], Gend = gam[ST - 1];
        *reinterpret_cast<float2 *>(&sm.gref[a1][c0]) = Gref;
        // per-(sub-tile, channel) factors; every product below stays in [e^-80, e^40]
        const float2 f1 = make_float2(exp2f(Ba.x - Gref.x), exp2f(Ba.y - Gref.y));      // >= 1
        const float2 f2 = make_float2(exp2f(Gref.x - Gend.x), exp2f(Gref.y - Gend.y));  // >= 1
        const float2 eB = make_float2(exp2f(Ba.x), exp2f(Ba.y));                        // <= 1
        const float2 fC = make_float2(exp2f(GC.x - Gend.x), exp2f(GC.y - Gend.y));      // <= 1
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const int r = a1 * ST + j;
            const float2 E1 = make_float2(exp2f(gam[j].x - Ba.x), exp2f(gam[j].y - Ba.y));
            const float2 E2 = make_float2(exp2f(Gend.x - gam[j].x), exp2f(Gend.y - gam[j].y));
            const float2 kf =
                unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.kL + r * LD + c0));
            const float2 qf =
                unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.qL + r * LD + c0));
            *reinterpret_cast<uint32_t *>(sm.kL + r * LD + c0) =
                pack_bf16x2(kf.x * E1.x * f1.x, kf.y * E1.y * f1.y);
            *reinterpret_cast<uint32_t *>(sm.qL + r * LD + c0) =
                pack_bf16x2(qf.x * E1.x * f1.x, qf.y * E1.y * f1.y);
            *reinterpret_cast<uint32_t *>(sm.kR + r * LD + c0) =
                pack_bf16x2(kf.x * E2.x * f2.x, kf.y * E2.y * f2.y);
            *reinterpret_cast<uint32_t *>(sm.kG + r * LD + c0) =
                pack_bf16x2(kf.x * E1.x * eB.x, kf.y * E1.y * eB.y);
            *reinterpret_cast<uint32_t *>(rec + REC_QG + swz128(r, c0)) =
                pack_bf16x2(qf.x * E1.x * eB.x, qf.y * E1.y * eB.y);
            *reinterpret_cast<uint32_t *>(rec + REC_KT + swz128(r, c0)) =
                pack_bf16x2(kf.x * E2.x * fC.x, kf.y * E2.y * fC.y);
        }
        if (a1 == NST - 1)
            *reinterpret_cast<float2 *>(rec + REC_GC + c0 * 4) =
                make_float2(exp2f(GC.x), exp2f(GC.y));
    }
    __syncthreads();

    // ---- P2: A blocks.  warp -> (row sub-tile a, kind: 0 keys, 1 queries) ----
    {
        const int a = warp >> 1, kind = warp & 1;
        const __nv_bfloat16 *left = kind ? sm.qL : sm.kL;
        for (int b = 0; b <= a; ++b) {
            float acc[2][4] = {};
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t af[4], bfr[4];
                ldsm_x4(af, smem_u32(left + (a * ST + frag_a_row(lane)) * LD + ks * 16 +
                                     frag_a_col(lane)));
                ldsm_x4(bfr, smem_u32(sm.kR + (b * ST + frag_bn_row(lane)) * LD + ks * 16 +
                                      frag_bn_col(lane)));
                if (b < a) {
                    // right rows of sub-tile b move their reference from G_ref(b) to G_ref(a)
                    const int cc = ks * 16 + 2 * tig;
                    const float m0 = exp2f(sm.gref[a][cc] - sm.gref[b][cc]);
                    const float m1 = exp2f(sm.gref[a][cc + 1] - sm.gref[b][cc + 1]);
                    const float m8 = exp2f(sm.gref[a][cc + 8] - sm.gref[b][cc + 8]);
                    const float m9 = exp2f(sm.gref[a][cc + 9] - sm.gref[b][cc + 9]);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 x = unpack_bf16x2(bfr[u]);
                        bfr[u] = (u & 1) ? pack_bf16x2(x.x * m8, x.y * m9)
                                         : pack_bf16x2(x.x * m0, x.y * m1);
                    }
                }
                mma_bf16_16816(acc[0], af, bfr[0], bfr[1]);
                mma_bf16_16816(acc[1], af, bfr[2], bfr[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rl = gid + 8 * hh, r = a * ST + rl;
                    const int il = nt * 8 + 2 * tig, i = b * ST + il;
                    float x0 = acc[nt][2 * hh], x1 = acc[nt][2 * hh + 1];
                    if (kind == 0) {
                        const float br = sm.beta[r];
                        if (b == a) {
                            sm.akd[a][rl][il] = (il < rl) ? x0 * br : 0.f;
                            sm.akd[a][rl][il + 1] = (il + 1 < rl) ? x1 * br : 0.f;
                        } else {
                            *reinterpret_cast<uint32_t *>(sm.akkn + r * LDA + i) =
                                pack_bf16x2(-x0 * br, -x1 * br);
                        }
                    } else {
                        if (b == a) {
                            x0 = (il <= rl) ? x0 : 0.f;
                            x1 = (il + 1 <= rl) ? x1 : 0.f;
                        }
                        *reinterpret_cast<uint32_t *>(rec + REC_AQK + swz64(r, i)) =
                            pack_bf16x2(x0, x1);
                    }
                }
        }
    }
    __syncthreads();

    // ---- P3: inverses of the 16x16 unit-lower diagonal blocks, fp32 ----
    if (tid < C) {
        const int a = tid >> 4, j = tid & 15;   // block a, column j: solve (I + A_aa) x = e_j
        float x[ST];
#pragma unroll
        for (int r = 0; r < ST; ++r) {
            float s = (r == j) ? 1.f : 0.f;
            if (r > j) {
#pragma unroll
                for (int i = 0; i < r; ++i)
                    if (i >= j) s -= sm.akd[a][r][i] * x[i];
            }
            x[r] = s;
        }
#pragma unroll
        for (int r = 0; r < ST; ++r) sm.taa[a][r * (ST + 8) + j] = f2bf(x[r]);
    }
    __syncthreads();

    // ---- P4: [W|U] by blocked forward substitution, warp-local column slices ----
    // warp w owns 32 columns: W[:, 32w..] (w < 4) or U[:, 32(w-4)..] (w >= 4).
    {
        __nv_bfloat16 *Y = sm.kL;                       // [C][LDY]: solution rows so far
        __nv_bfloat16 *Z = sm.kR + warp * (ST * 40);    // warp scratch [16][40]
        const __nv_bfloat16 *X = warp < 4 ? sm.kG : sm.v;
        const int xc = (warp & 3) * 32;                 // column base inside X / W / U
        const int yc = warp * 32;                       // column base inside Y
        for (int a = 0; a < NST; ++a) {
            float acc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = a * ST + gid + 8 * hh;
                    const float2 x = unpack_bf16x2(
                        *reinterpret_cast<const uint32_t *>(X + r * LD + xc + nt * 8 + 2 * tig));
                    acc[nt][2 * hh] = sm.beta[r] * x.x;
                    acc[nt][2 * hh + 1] = sm.beta[r] * x.y;
                }
            for (int b = 0; b < a; ++b) {   // acc -= A_ab Y_b  (akkn holds -A)
                uint32_t af[4];
                ldsm_x4(af, smem_u32(sm.akkn + (a * ST + frag_a_row(lane)) * LDA + b * ST +
                                     frag_a_col(lane)));
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    uint32_t bb[4];
                    ldsm_x4_t(bb, smem_u32(Y + (b * ST + frag_bk_row(lane)) * LDY + yc +
                                           np * 16 + frag_bk_col(lane)));
                    mma_bf16_16816(acc[2 * np], af, bb[0], bb[1]);
                    mma_bf16_16816(acc[2 * np + 1], af, bb[2], bb[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint32_t *>(Z + (gid + 8 * hh) * 40 + nt * 8 + 2 * tig) =
                        pack_bf16x2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
            __syncwarp();
            float y[4][4] = {};
            uint32_t at[4];
            ldsm_x4(at, smem_u32(sm.taa[a] + frag_a_row(lane) * (ST + 8) + frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bz[4];
                ldsm_x4_t(bz, smem_u32(Z + frag_bk_row(lane) * 40 + np * 16 + frag_bk_col(lane)));
                mma_bf16_16816(y[2 * np], at, bz[0], bz[1]);
                mma_bf16_16816(y[2 * np + 1], at, bz[2], bz[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = a * ST + gid + 8 * hh;
                    const int cl = nt * 8 + 2 * tig;
                    const uint32_t pk = pack_bf16x2(y[nt][2 * hh], y[nt][2 * hh + 1]);
                    *reinterpret_cast<uint32_t *>(Y + r * LDY + yc + cl) = pk;
                    if (warp < 4)
                        *reinterpret_cast<uint32_t *>(rec + REC_W + swz128(r, xc + cl)) = pk;
                    else
                        *reinterpret_cast<uint32_t *>(rec + rec_u_off(r, xc + cl)) = pk;
                }
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: inter-chunk state pass.  grid = N * H * (D / DVT), 256 threads.
// Warp w owns key rows 16w..16w+15 of the fp32 state tile S[:, col0:col0+DVT],
// held in MMA accumulator registers; a bf16 copy in smem feeds W S and Qg S.
// Chunk records arrive by bulk copies into a 3-stage mbarrier ring; every wait
// is bounded (a wait that runs out sets the timeout bit and the CTA returns).
// ---------------------------------------------------------------------------
constexpr int NSTAGE = 3;

template <int DVT>
struct StateSmem {
    static constexpr int STAGE_BYTES = REC_SHARED + C * DVT * 2;
    uint8_t stage[NSTAGE][STAGE_BYTES];        // [W|Kt|Qg|Aqk|gC] + U tile(s)
    __nv_bfloat16 sb[D * (DVT + 8)];           // bf16 copy of the state tile
    __nv_bfloat16 db[C * (DVT + 8)];           // bf16 Delta tile
    uint64_t full[NSTAGE];
};

template <int DVT>
__global__ void __launch_bounds__(256, 1)
kda_tc_state_kernel(const uint8_t *__restrict__ recs, const float *h0, float *hT,
                    __nv_bfloat16 *__restrict__ o, int T, int H, int cps,
                    const int *__restrict__ hdr, const int *__restrict__ seq_off,
                    const int *__restrict__ cu, int *err_word, int debug_drop_first_copy) {
    constexpr int NT = DVT / 8;    // n-tiles of the column tile
    constexpr int LDV = DVT + 8;
    constexpr int STAGE_BYTES = StateSmem<DVT>::STAGE_BYTES;
    static_assert(STAGE_BYTES % 128 == 0, "stage alignment");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    StateSmem<DVT> &sm = *reinterpret_cast<StateSmem<DVT> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // 1-D grid, column tile fastest so the tiles of one chain run side by side
    // and share the chunk records through L2.
    const int tile = blockIdx.x % (D / DVT), col0 = tile * DVT;
    const int chain = blockIdx.x / (D / DVT), n = chain / H, h = chain % H;

    int c_begin, c_end, seq_t0, seq_len;
    if (cu) {
        if (!hdr[0]) return;
        c_begin = seq_off[n];
        c_end = seq_off[n + 1];
        seq_t0 = cu[n];
        seq_len = cu[n + 1] - cu[n];
    } else {
        c_begin = n * cps;
        c_end = c_begin + cps;
        seq_t0 = n * T;
        seq_len = T;
    }
    const int nchunks = c_end - c_begin;

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    auto issue = [&](int j) {   // thread 0 only: bring chunk j into stage j % NSTAGE
        uint64_t *bar = &sm.full[j % NSTAGE];
        const uint8_t *rec = recs + ((size_t)(c_begin + j) * H + h) * REC_BYTES;
        uint8_t *dst = sm.stage[j % NSTAGE];
        mbar_arrive_expect_tx(bar, STAGE_BYTES);
        if (debug_drop_first_copy && j == 0) return;   // test hook: the wait must run out
        bulk_g2s(dst, rec, REC_SHARED, bar);
        bulk_g2s(dst + REC_SHARED, rec + REC_U + tile * (C * DVT * 2), C * DVT * 2, bar);
    };
    if (tid == 0)
        for (int j = 0; j < NSTAGE && j < nchunks; ++j) issue(j);

    // state rows 16w..16w+15 -> accumulator registers
    float S[NT][4];
    const size_t sbase = (size_t)chain * D * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = warp * 16 + gid + 8 * hh;
            const int col = col0 + nt * 8 + 2 * tig;
            float2 x = make_float2(0.f, 0.f);
            if (h0) x = *reinterpret_cast<const float2 *>(h0 + sbase + (size_t)r * D + col);
            S[nt][2 * hh] = x.x;
            S[nt][2 * hh + 1] = x.y;
        }
    auto store_sb = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + gid + 8 * hh;
                *reinterpret_cast<uint32_t *>(sm.sb + r * LDV + nt * 8 + 2 * tig) =
                    pack_bf16x2(S[nt][2 * hh], S[nt][2 * hh + 1]);
            }
    };
    store_sb();
    __syncthreads();

    for (int j = 0; j < nchunks; ++j) {
        const int s = j % NSTAGE;
        if (!mbar_wait_bounded(&sm.full[s], (j / NSTAGE) & 1)) {
            // Give up on this chain: report, let the copies already issued for later
            // chunks land (bounded) so none writes into freed shared memory, return.
            if (tid == 0) {
                atomicOr(err_word, ERR_TIMEOUT_BIT);
                for (int jj = j + 1; jj < j + NSTAGE && jj < nchunks; ++jj)
                    mbar_wait_bounded(&sm.full[jj % NSTAGE], (jj / NSTAGE) & 1);
            }
            return;
        }
        const uint8_t *st = sm.stage[s];
        const uint32_t sW = smem_u32(st + REC_W), sKt = smem_u32(st + REC_KT);
        const uint32_t sQg = smem_u32(st + REC_QG), sA = smem_u32(st + REC_AQK);
        const float *gc = reinterpret_cast<const float *>(st + REC_GC);
        const __nv_bfloat16 *u = reinterpret_cast<const __nv_bfloat16 *>(st + REC_SHARED);
        const int t0 = seq_t0 + j * C;
        const int len = min(C, seq_len - j * C);

        // Phase A: warps 0-3 -> Delta = U - W S (rows 16w..), warps 4-7 -> Oq = Qg S
        const int rw = (warp & 3) * 16;
        const uint32_t sL = warp < 4 ? sW : sQg;
        float P[NT][4] = {};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t af[4];
            ldsm_x4(af, sL + swz128(rw + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b[4];
                ldsm_x4_t(b, smem_u32(sm.sb + (ks * 16 + frag_bk_row(lane)) * LDV + np * 16 +
                                      frag_bk_col(lane)));
                mma_bf16_16816(P[2 * np], af, b[0], b[1]);
                mma_bf16_16816(P[2 * np + 1], af, b[2], b[3]);
            }
        }
        if (warp < 4) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = rw + gid + 8 * hh;
                    const int cl = nt * 8 + 2 * tig;
                    const float2 uu = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
                        u + (cl >> 4) * (C * UT) + r * UT + (cl & 15)));
                    *reinterpret_cast<uint32_t *>(sm.db + r * LDV + cl) =
                        pack_bf16x2(uu.x - P[nt][2 * hh], uu.y - P[nt][2 * hh + 1]);
                }
        }
        __syncthreads();

        // Phase B: all warps update their 16 state rows: S = Diag(exp G_C) S + Kt^T Delta
        {
            const float g0 = gc[warp * 16 + gid], g8 = gc[warp * 16 + gid + 8];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                S[nt][0] *= g0;
                S[nt][1] *= g0;
                S[nt][2] *= g8;
                S[nt][3] *= g8;
            }
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                uint32_t ak[4];
                ldsm_x4_t(ak, sKt + swz128(ks * 16 + frag_at_row(lane),
                                           warp * 16 + frag_at_col(lane)));
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    uint32_t bd[4];
                    ldsm_x4_t(bd, smem_u32(sm.db + (ks * 16 + frag_bk_row(lane)) * LDV +
                                           np * 16 + frag_bk_col(lane)));
                    mma_bf16_16816(S[2 * np], ak, bd[0], bd[1]);
                    mma_bf16_16816(S[2 * np + 1], ak, bd[2], bd[3]);
                }
            }
        }
        // warps 4-7: O = Qg S + Aqk Delta (lower triangular: k-steps 0..rw/16)
        if (warp >= 4) {
            const int wr = warp - 4;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                if (ks <= wr) {
                    uint32_t aa[4];
                    ldsm_x4(aa, sA + swz64(rw + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t bd[4];
                        ldsm_x4_t(bd, smem_u32(sm.db + (ks * 16 + frag_bk_row(lane)) * LDV +
                                               np * 16 + frag_bk_col(lane)));
                        mma_bf16_16816(P[2 * np], aa, bd[0], bd[1]);
                        mma_bf16_16816(P[2 * np + 1], aa, bd[2], bd[3]);
                    }
                }
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = rw + gid + 8 * hh;
                if (r < len) {
                    __nv_bfloat16 *orow = o + ((size_t)(t0 + r) * H + h) * D + col0;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        *reinterpret_cast<uint32_t *>(orow + nt * 8 + 2 * tig) =
                            pack_bf16x2(P[nt][2 * hh], P[nt][2 * hh + 1]);
                }
            }
        }
        store_sb();
        __syncthreads();   // state copy ready; stage s and db free
        if (tid == 0 && j + NSTAGE < nchunks) {
            fence_proxy_async_smem();   // order this chunk's generic reads before the refill
            issue(j + NSTAGE);
        }
    }

    if (hT) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + gid + 8 * hh;
                const int col = col0 + nt * 8 + 2 * tig;
                *reinterpret_cast<float2 *>(hT + sbase + (size_t)r * D + col) =
                    make_float2(S[nt][2 * hh], S[nt][2 * hh + 1]);
            }
    }
}

}  // namespace tc
}  // namespace kda
