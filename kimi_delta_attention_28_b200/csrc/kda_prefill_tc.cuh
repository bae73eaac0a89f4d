// kda_prefill_tc.cuh -- chunkwise KDA prefill on tensor cores, bf16 q/k/v, d_k = d_v = 128.
//
// The recurrence (single head, "Kimi K3" open-weights field notes, panel
// "KDA 单头递归"):  S_t = (I - b_t k_t k_t^T) Diag(exp g_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t.  Over a chunk of C tokens with inclusive cumulative log-decay
// G_r (per key channel), unrolling the recurrence gives the exact chunk form
//
//   A_ri  = b_r sum_c k_rc k_ic exp(G_rc - G_ic)      (i < r, strictly lower)
//   T     = (I + A)^-1,  W = T Diag(b) (K * exp G),  U = T Diag(b) V
//   Delta = U - W S_in                                (per-token delta-rule errors)
//   O     = (Q * exp G) S_in + [i <= r](sum_c q_rc k_ic exp(G_rc - G_ic)) Delta
//   S_out = Diag(exp G_C) S_in + (K * exp(G_C - G))^T Delta
//
// Kernel 1 (kda_tc_prep_kernel) computes every chunk-local quantity, fully in
// parallel over (chunk, head): the log-decay cumsum, A (with the pairwise decays
// factored through 16-token sub-tile reference points so no factor overflows:
// the same page's panel "g ∈ (-5, 0)" bounds a 16-token decay by e^-80), the
// triangular inverse, W, U, the decayed keys/queries and the masked query-key
// block.  Kernel 2 (kda_tc_state_kernel) walks the chunks of each (sequence,
// head) in order with the fp32 state resident on chip, split over d_v column
// tiles (state columns evolve independently), and writes o and the final state.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace tc {

constexpr int D = 128;          // head size (d_k = d_v)
constexpr int C = 64;           // chunk length
constexpr int ST = 16;          // sub-tile length for the decay reference points
constexpr int NST = C / ST;     // sub-tiles per chunk
constexpr int LD = D + 8;       // padded bf16 row stride (272 B: conflict-free ldmatrix)
constexpr int LDA = C + 4;      // fp32 row stride of the A matrix in smem
constexpr int LDT = C + 8;      // padded bf16 row stride of T' and the query-key block

// Per (chunk, head) record written by kernel 1 and read by kernel 2.
constexpr int REC_W = 0;                       // W       [C][D] bf16
constexpr int REC_U = REC_W + C * D * 2;       // U       [C][D] bf16
constexpr int REC_KT = REC_U + C * D * 2;      // K*exp(G_C - G)  [C][D] bf16
constexpr int REC_QG = REC_KT + C * D * 2;     // Q*exp(G)        [C][D] bf16
constexpr int REC_AQK = REC_QG + C * D * 2;    // masked query-key block [C][C] bf16
constexpr int REC_GC = REC_AQK + C * C * 2;    // exp(G_C)        [D] fp32
constexpr int REC_BYTES = REC_GC + D * 4;      // 74240 (a multiple of 256)
static_assert(REC_BYTES % 256 == 0, "record alignment");

// Workspace header: [0] = offsets valid (1) / invalid (0), [1] = total chunks.
struct ChunkLoc {
    int t0;    // first token (flattened over the batch / packed sequences)
    int len;   // tokens in this chunk, 1..C
};

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
    __nv_bfloat16 kL[C * LD];    // raw k, then k*exp(G_r - G_mid)       (A left, keys)
    __nv_bfloat16 qL[C * LD];    // raw q, then q*exp(G_r - G_mid); later fp32 T scratch
    __nv_bfloat16 v[C * LD];     // raw v
    __nv_bfloat16 kR[C * LD];    // k*exp(G_mid - G_i)                    (A right); later X scratch
    __nv_bfloat16 kG[C * LD];    // k*exp(G_r)                            (for W)
    float akk[C * LDA];          // b_r * A_ri (strictly lower)
    float gmid[NST][D];          // G at each sub-tile's reference row (log2 units)
    float xch[2][D];             // half-chunk decay totals
    float beta[C];
};

__global__ void __launch_bounds__(256, 2)
kda_tc_prep_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                   const __nv_bfloat16 *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, int T, int H, int cps,
                   const int *__restrict__ hdr, const ChunkLoc *__restrict__ chunks,
                   uint8_t *__restrict__ recs) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    for (int i = tid; i < 3 * C * (D / 8); i += 256) {
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

    // ---- P1: per-channel cumulative decay and the scaled operands ----
    // thread -> channel c, rows [32*half, 32*half + 32).  Work in log2 units.
    const int c = tid & (D - 1), half = tid >> 7;
    float gam[32];
    {
        float run = 0.f;
        const float *gp = g + base + c;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = half * 32 + i;
            const float gv = r < len ? gp[r * rowstride] : 0.f;
            run += gv * kLog2e;
            gam[i] = run;
        }
        sm.xch[half][c] = run;
    }
    cp_async_wait<0>();
    __syncthreads();
    const float off = half ? sm.xch[0][c] : 0.f;
    const float gC = sm.xch[0][c] + sm.xch[1][c];
#pragma unroll
    for (int i = 0; i < 32; ++i) gam[i] += off;
    __nv_bfloat16 *gKt = reinterpret_cast<__nv_bfloat16 *>(rec + REC_KT);
    __nv_bfloat16 *gQg = reinterpret_cast<__nv_bfloat16 *>(rec + REC_QG);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int a = 2 * half + s;
        const float Ba = (s == 0) ? off : gam[15];       // G at row 16a - 1
        const float Gend = gam[16 * s + 15], Gmid = gam[16 * s + 7];
        sm.gmid[a][c] = Gmid;
        const float f1 = exp2f(Ba - Gmid);    // >= 1, <= e^40
        const float f2 = exp2f(Gmid - Gend);  // >= 1, <= e^40
        const float eB = exp2f(Ba);           // <= 1
        const float fC = exp2f(gC - Gend);    // <= 1
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const int r = a * ST + j;
            const float G = gam[16 * s + j];
            const float E1 = exp2f(G - Ba);    // in [e^-80, 1]
            const float E2 = exp2f(Gend - G);  // in [e^-80, 1]
            const float kf = bf2f(sm.kL[r * LD + c]);
            const float qf = bf2f(sm.qL[r * LD + c]);
            sm.kL[r * LD + c] = f2bf(kf * E1 * f1);
            sm.qL[r * LD + c] = f2bf(qf * E1 * f1);
            sm.kR[r * LD + c] = f2bf(kf * E2 * f2);
            sm.kG[r * LD + c] = f2bf(kf * E1 * eB);
            gQg[r * D + c] = f2bf(qf * E1 * eB);
            gKt[r * D + c] = f2bf(kf * E2 * fC);
        }
    }
    if (half == 1) reinterpret_cast<float *>(rec + REC_GC)[c] = exp2f(gC);
    __syncthreads();

    // ---- P2: A blocks.  warp -> (row sub-tile a, kind: 0 keys, 1 queries) ----
    {
        const int a = warp >> 1, kind = warp & 1;
        const int gid = lane >> 2, tig = lane & 3;
        const __nv_bfloat16 *left = kind ? sm.qL : sm.kL;
        __nv_bfloat16 *gAqk = reinterpret_cast<__nv_bfloat16 *>(rec + REC_AQK);
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
                    // right rows of sub-tile b move their reference from G_mid(b) to G_mid(a)
                    const int c0 = ks * 16 + 2 * tig;
                    const float m0 = exp2f(sm.gmid[a][c0] - sm.gmid[b][c0]);
                    const float m1 = exp2f(sm.gmid[a][c0 + 1] - sm.gmid[b][c0 + 1]);
                    const float m8 = exp2f(sm.gmid[a][c0 + 8] - sm.gmid[b][c0 + 8]);
                    const float m9 = exp2f(sm.gmid[a][c0 + 9] - sm.gmid[b][c0 + 9]);
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
                    const int r = a * ST + gid + 8 * hh;
                    const int i = b * ST + nt * 8 + 2 * tig;
                    float x0 = acc[nt][2 * hh], x1 = acc[nt][2 * hh + 1];
                    if (kind == 0) {
                        const float br = sm.beta[r];
                        if (b == a) {
                            x0 = (i < r) ? x0 : 0.f;
                            x1 = (i + 1 < r) ? x1 : 0.f;
                        }
                        sm.akk[r * LDA + i] = x0 * br;
                        sm.akk[r * LDA + i + 1] = x1 * br;
                    } else {
                        if (b == a) {
                            x0 = (i <= r) ? x0 : 0.f;
                            x1 = (i + 1 <= r) ? x1 : 0.f;
                        }
                        *reinterpret_cast<uint32_t *>(gAqk + r * C + i) = pack_bf16x2(x0, x1);
                    }
                }
        }
    }
    __syncthreads();

    // ---- P3: T = (I + A)^-1 in fp32 (blocked forward substitution) ----
    float *Tf = reinterpret_cast<float *>(sm.qL);  // [C][C] fp32, 16 KB (fits in qL)
    float *X = reinterpret_cast<float *>(sm.kR);   // [3][16][16] fp32 scratch
    if (tid < C) {
        // diagonal block a, column j: solve (I + A_aa) x = e_j
        const int a = tid >> 4, j = tid & 15;
        float x[ST];
#pragma unroll
        for (int r = 0; r < ST; ++r) {
            float s = (r == j) ? 1.f : 0.f;
            if (r > j) {
#pragma unroll
                for (int i = 0; i < r; ++i)
                    if (i >= j) s -= sm.akk[(a * ST + r) * LDA + a * ST + i] * x[i];
            }
            x[r] = s;
        }
#pragma unroll
        for (int r = 0; r < ST; ++r) Tf[(a * ST + r) * C + a * ST + j] = x[r];
    }
    __syncthreads();
    for (int d = 1; d < NST; ++d) {
        const int nblk = NST - d;
        // X_ab = sum_{j=b}^{a-1} A_aj T_jb
        for (int e = tid; e < nblk * ST * ST; e += 256) {
            const int blk = e / (ST * ST), r = (e / ST) % ST, s = e % ST;
            const int a = d + blk, b = a - d;
            float acc = 0.f;
            for (int jj = b * ST; jj < a * ST; ++jj)
                acc += sm.akk[(a * ST + r) * LDA + jj] * Tf[jj * C + b * ST + s];
            X[e] = acc;
        }
        __syncthreads();
        // T_ab = -T_aa X_ab
        for (int e = tid; e < nblk * ST * ST; e += 256) {
            const int blk = e / (ST * ST), r = (e / ST) % ST, s = e % ST;
            const int a = d + blk, b = a - d;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i)
                acc += Tf[(a * ST + r) * C + a * ST + i] * X[blk * ST * ST + i * ST + s];
            Tf[(a * ST + r) * C + b * ST + s] = -acc;
        }
        __syncthreads();
    }
    // T' = T Diag(beta) in bf16 (zero above the diagonal), into the kL slot.
    __nv_bfloat16 *Tb = sm.kL;  // [C][LDT]
    for (int e = tid; e < C * C; e += 256) {
        const int r = e / C, i = e % C;
        Tb[r * LDT + i] = f2bf(i <= r ? Tf[r * C + i] * sm.beta[i] : 0.f);
    }
    __syncthreads();

    // ---- P4: W = T' (K*exp G), U = T' V ----
    {
        const int mt = warp & 3, ch = warp >> 2;
        const int gid = lane >> 2, tig = lane & 3;
        float accW[8][4] = {}, accU[8][4] = {};
        for (int ks = 0; ks <= mt; ++ks) {
            uint32_t af[4];
            ldsm_x4(af, smem_u32(Tb + (mt * 16 + frag_a_row(lane)) * LDT + ks * 16 +
                                 frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bw[4], bu[4];
                const int col = ch * 64 + np * 16 + frag_bk_col(lane);
                const int row = ks * 16 + frag_bk_row(lane);
                ldsm_x4_t(bw, smem_u32(sm.kG + row * LD + col));
                ldsm_x4_t(bu, smem_u32(sm.v + row * LD + col));
                mma_bf16_16816(accW[2 * np], af, bw[0], bw[1]);
                mma_bf16_16816(accW[2 * np + 1], af, bw[2], bw[3]);
                mma_bf16_16816(accU[2 * np], af, bu[0], bu[1]);
                mma_bf16_16816(accU[2 * np + 1], af, bu[2], bu[3]);
            }
        }
        __nv_bfloat16 *gW = reinterpret_cast<__nv_bfloat16 *>(rec + REC_W);
        __nv_bfloat16 *gU = reinterpret_cast<__nv_bfloat16 *>(rec + REC_U);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = mt * 16 + gid + 8 * hh;
                const int col = ch * 64 + nt * 8 + 2 * tig;
                *reinterpret_cast<uint32_t *>(gW + r * D + col) =
                    pack_bf16x2(accW[nt][2 * hh], accW[nt][2 * hh + 1]);
                *reinterpret_cast<uint32_t *>(gU + r * D + col) =
                    pack_bf16x2(accU[nt][2 * hh], accU[nt][2 * hh + 1]);
            }
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: inter-chunk state pass.  grid = N * H * (D / DVT), 128 threads.
// The fp32 state tile S[:, col0:col0+DVT] lives in MMA accumulator registers
// (warp w owns key rows 32w..32w+31); a bf16 copy in smem feeds W S and Qg S.
// ---------------------------------------------------------------------------
template <int DVT>
struct StateStage {
    __nv_bfloat16 w[C * LD];
    __nv_bfloat16 kt[C * LD];
    __nv_bfloat16 qg[C * LD];
    __nv_bfloat16 aqk[C * LDT];
    __nv_bfloat16 u[C * (DVT + 8)];
    float gc[D];
};
template <int DVT>
struct StateSmem {
    StateStage<DVT> st[2];
    __nv_bfloat16 sb[D * (DVT + 8)];     // bf16 copy of the state tile
    __nv_bfloat16 db[C * (DVT + 8)];     // bf16 Delta tile
};

template <int DVT>
__device__ __forceinline__ void state_prefetch(StateStage<DVT> &st, const uint8_t *rec, int col0,
                                               int tid) {
    constexpr int LDV = DVT + 8;
    // W, Kt, Qg: 3 x 64 rows x 16 chunks of 16 B
    for (int i = tid; i < 3 * C * (D / 8); i += 128) {
        const int m = i / (C * (D / 8)), rem = i % (C * (D / 8));
        const int r = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
        const int off = (m == 0 ? REC_W : (m == 1 ? REC_KT : REC_QG));
        __nv_bfloat16 *dst = (m == 0 ? st.w : (m == 1 ? st.kt : st.qg)) + r * LD + c8;
        cp_async16(dst, rec + off + (r * D + c8) * 2);
    }
    for (int i = tid; i < C * (C / 8); i += 128) {
        const int r = i / (C / 8), c8 = (i % (C / 8)) * 8;
        cp_async16(st.aqk + r * LDT + c8, rec + REC_AQK + (r * C + c8) * 2);
    }
    for (int i = tid; i < C * (DVT / 8); i += 128) {
        const int r = i / (DVT / 8), c8 = (i % (DVT / 8)) * 8;
        cp_async16(st.u + r * LDV + c8, rec + REC_U + (r * D + col0 + c8) * 2);
    }
    if (tid < D / 4) cp_async16(st.gc + tid * 4, rec + REC_GC + tid * 16);
}

template <int DVT>
__global__ void __launch_bounds__(128, 1)
kda_tc_state_kernel(const uint8_t *__restrict__ recs, const float *h0,
                    float *hT, __nv_bfloat16 *__restrict__ o, int T, int H, int cps,
                    const int *__restrict__ hdr, const int *__restrict__ seq_off,
                    const int *__restrict__ cu) {
    constexpr int NT = DVT / 8;    // n-tiles of the column tile
    constexpr int LDV = DVT + 8;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    StateSmem<DVT> &sm = *reinterpret_cast<StateSmem<DVT> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    // 1-D grid, column tile fastest so the tiles of one chain run side by side
    // and share the chunk records through L2.
    const int col0 = (blockIdx.x % (D / DVT)) * DVT;
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

    // state tile -> accumulator registers
    float S[2][NT][4];
    const size_t sbase = (size_t)chain * D * D;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 32 + mt * 16 + gid + 8 * hh;
                const int col = col0 + nt * 8 + 2 * tig;
                float2 x = make_float2(0.f, 0.f);
                if (h0) x = *reinterpret_cast<const float2 *>(h0 + sbase + (size_t)r * D + col);
                S[mt][nt][2 * hh] = x.x;
                S[mt][nt][2 * hh + 1] = x.y;
            }
    auto store_sb = [&]() {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = warp * 32 + mt * 16 + gid + 8 * hh;
                    *reinterpret_cast<uint32_t *>(sm.sb + r * LDV + nt * 8 + 2 * tig) =
                        pack_bf16x2(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                }
    };
    store_sb();

    const int nchunks = c_end - c_begin;
    if (nchunks > 0) {
        state_prefetch<DVT>(sm.st[0], recs + ((size_t)c_begin * H + h) * REC_BYTES, col0, tid);
    }
    cp_async_commit();

    for (int j = 0; j < nchunks; ++j) {
        if (j + 1 < nchunks)
            state_prefetch<DVT>(sm.st[(j + 1) & 1],
                                recs + ((size_t)(c_begin + j + 1) * H + h) * REC_BYTES, col0, tid);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const StateStage<DVT> &st = sm.st[j & 1];
        const int t0 = seq_t0 + j * C;
        const int len = min(C, seq_len - j * C);

        // Delta = U - W S and the inter-chunk output term Qg S, rows 16w..16w+15
        float P[NT][4] = {}, Oq[NT][4] = {};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t aw[4], aq[4];
            ldsm_x4(aw, smem_u32(st.w + (warp * 16 + frag_a_row(lane)) * LD + ks * 16 +
                                 frag_a_col(lane)));
            ldsm_x4(aq, smem_u32(st.qg + (warp * 16 + frag_a_row(lane)) * LD + ks * 16 +
                                 frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b[4];
                ldsm_x4_t(b, smem_u32(sm.sb + (ks * 16 + frag_bk_row(lane)) * LDV + np * 16 +
                                      frag_bk_col(lane)));
                mma_bf16_16816(P[2 * np], aw, b[0], b[1]);
                mma_bf16_16816(P[2 * np + 1], aw, b[2], b[3]);
                mma_bf16_16816(Oq[2 * np], aq, b[0], b[1]);
                mma_bf16_16816(Oq[2 * np + 1], aq, b[2], b[3]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + gid + 8 * hh;
                const float2 u = unpack_bf16x2(
                    *reinterpret_cast<const uint32_t *>(st.u + r * LDV + nt * 8 + 2 * tig));
                *reinterpret_cast<uint32_t *>(sm.db + r * LDV + nt * 8 + 2 * tig) =
                    pack_bf16x2(u.x - P[nt][2 * hh], u.y - P[nt][2 * hh + 1]);
            }
        __syncthreads();

        // Delta as B fragments for all four 16-row k-steps
        uint32_t bd[C / 16][NT / 2][4];
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
#pragma unroll
            for (int np = 0; np < NT / 2; ++np)
                ldsm_x4_t(bd[ks][np], smem_u32(sm.db + (ks * 16 + frag_bk_row(lane)) * LDV +
                                               np * 16 + frag_bk_col(lane)));

        // O = Qg S + Aqk Delta (Aqk lower triangular: k-steps 0..warp)
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
            if (ks <= warp) {
                uint32_t aa[4];
                ldsm_x4(aa, smem_u32(st.aqk + (warp * 16 + frag_a_row(lane)) * LDT + ks * 16 +
                                     frag_a_col(lane)));
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    mma_bf16_16816(Oq[2 * np], aa, bd[ks][np][0], bd[ks][np][1]);
                    mma_bf16_16816(Oq[2 * np + 1], aa, bd[ks][np][2], bd[ks][np][3]);
                }
            }
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = warp * 16 + gid + 8 * hh;
            if (r < len) {
                __nv_bfloat16 *orow = o + ((size_t)(t0 + r) * H + h) * D + col0;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    *reinterpret_cast<uint32_t *>(orow + nt * 8 + 2 * tig) =
                        pack_bf16x2(Oq[nt][2 * hh], Oq[nt][2 * hh + 1]);
            }
        }

        // S = Diag(exp G_C) S + Kt^T Delta for key rows 32w..32w+31
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const float g0 = st.gc[warp * 32 + mt * 16 + gid];
            const float g8 = st.gc[warp * 32 + mt * 16 + gid + 8];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                S[mt][nt][0] *= g0;
                S[mt][nt][1] *= g0;
                S[mt][nt][2] *= g8;
                S[mt][nt][3] *= g8;
            }
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                uint32_t ak[4];
                ldsm_x4_t(ak, smem_u32(st.kt + (ks * 16 + frag_at_row(lane)) * LD + warp * 32 +
                                       mt * 16 + frag_at_col(lane)));
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    mma_bf16_16816(S[mt][2 * np], ak, bd[ks][np][0], bd[ks][np][1]);
                    mma_bf16_16816(S[mt][2 * np + 1], ak, bd[ks][np][2], bd[ks][np][3]);
                }
            }
        }
        store_sb();
        __syncthreads();
    }

    if (hT) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = warp * 32 + mt * 16 + gid + 8 * hh;
                    const int col = col0 + nt * 8 + 2 * tig;
                    *reinterpret_cast<float2 *>(hT + sbase + (size_t)r * D + col) =
                        make_float2(S[mt][nt][2 * hh], S[mt][nt][2 * hh + 1]);
                }
    }
}

}  // namespace tc
}  // namespace kda
