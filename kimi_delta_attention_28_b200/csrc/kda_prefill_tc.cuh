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
// of the 16x16 diagonal blocks, tensor-core products elsewhere); and from them
// the chunk's affine map on the state (below), one record per (chunk, head).
// Kernel 2 (kda_tc_state_kernel) walks the chunks of each (sequence, head) in
// order with the fp32 state on chip, split over d_v column tiles (state columns
// evolve independently), one product chain per chunk; records arrive by bulk
// copies into a 3-stage ring.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace tc {

constexpr int D = 128;          // head size (d_k = d_v)
constexpr int C = 64;           // chunk length
constexpr int ST = 16;          // sub-tile length for the decay reference rows
constexpr int NST = C / ST;     // sub-tiles per chunk

// Per (chunk, head) record, written by kernel 1 and read by kernel 2: the
// chunk's affine map.  With W, U, Kt = K*exp(G_C - G), Qg = Q*exp(G) and the
// masked query-key block Aqk, a chunk takes the state S_in to
//   S_out = Diag(exp G_C) S_in + M' S_in + R,   M' = -Kt^T W,  R = Kt^T U
//   O     = Q' S_in + O0,                      Q' = Qg - Aqk W,  O0 = Aqk U
// [rows][128] tiles use the swz128 layout (16-byte chunks XOR-permuted by row)
// so a plain bulk copy lands them in shared memory ready for conflict-free
// ldmatrix; R and O0 are stored as 16-column tiles so each column slice of the
// state reads one contiguous block.
constexpr int REC_M = 0;                     // M'        [D][D] bf16, swz128
constexpr int REC_QP = REC_M + D * D * 2;    // Q'        [C][D] bf16, swz128
constexpr int REC_GC = REC_QP + C * D * 2;   // exp(G_C)  [D] fp32
constexpr int REC_SHARED = REC_GC + D * 4;   // bytes every column slice reads (49,664)
constexpr int UT = 16;                       // column tile width of R and O0
constexpr int REC_R = REC_SHARED;            // R   [D/UT][D][UT] bf16
constexpr int REC_O0 = REC_R + D * D * 2;    // O0  [D/UT][C][UT] bf16
constexpr int REC_BYTES = REC_O0 + C * D * 2;  // 98,816
// Kt and Qg pass through the R and O0 areas of the record (swz128) before
// those are written: kernel 1 needs them after its shared memory has been reused.
constexpr int REC_KT_SCRATCH = REC_R;
constexpr int REC_QG_SCRATCH = REC_O0;
static_assert(REC_BYTES % 256 == 0 && REC_SHARED % 16 == 0 && REC_O0 % 16 == 0, "alignment");

KDA_DEVINL int rec_r_off(int r, int c) {
    return REC_R + (c >> 4) * (D * UT * 2) + r * (UT * 2) + (c & 15) * 2;
}
KDA_DEVINL int rec_o0_off(int r, int c) {
    return REC_O0 + (c >> 4) * (C * UT * 2) + r * (UT * 2) + (c & 15) * 2;
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
constexpr int LDA = C + 8;      // padded bf16 row stride of the 64x64 blocks (144 B)
constexpr int ZLD = 40;         // row stride of the per-warp substitution scratch

// The six sub-tile pairs (a, b), b < a, of a 64-token chunk.
__constant__ int2 kPairs[6] = {{1, 0}, {2, 0}, {3, 0}, {2, 1}, {3, 1}, {3, 2}};

struct PrepSmem {
    // Five 16 KB tiles in swz128 layout, reused across phases:
    //   r0: k -> k*exp(G_r - G_ref(a)) ; then, with r1, the [W|U] solution (swz256)
    //   r1: q -> q*exp(G_r - G_ref(a))
    //   r2: v
    //   r3: k*exp(G_ref(b) - G_i) ; then per-warp scratch ; then Kt
    //   r4: k*exp(G_r) ; then Qg
    uint8_t r0[C * D * 2], r1[C * D * 2], r2[C * D * 2], r3[C * D * 2], r4[C * D * 2];
    __nv_bfloat16 akkn[C * LDA];   // -b_r A_ri, sub-tile blocks b < a (bf16)
    __nv_bfloat16 aqk[C * LDA];    // masked query-key block (bf16)
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
    const uint32_t s0 = smem_u32(sm.r0), s1 = smem_u32(sm.r1), s2 = smem_u32(sm.r2);
    const uint32_t s3 = smem_u32(sm.r3), s4 = smem_u32(sm.r4);

    // ---- P0: stage k, q, v rows (zero-filled past len) and beta ----
#pragma unroll
    for (int it = 0; it < 3 * C * (D / 8) / 256; ++it) {
        const int i = tid + it * 256;
        const int m = i / (C * (D / 8));
        const int rem = i % (C * (D / 8));
        const int r = rem / (D / 8), c8 = (rem % (D / 8)) * 8;
        const __nv_bfloat16 *src = (m == 0 ? k : (m == 1 ? q : v));
        uint8_t *dst = (m == 0 ? sm.r0 : (m == 1 ? sm.r1 : sm.r2)) + swz128(r, c8);
        const bool ok = r < len;
        cp_async16(dst, ok ? (src + base + r * rowstride + c8) : src, ok ? 16 : 0);
    }
    cp_async_commit();
    if (tid < C) sm.beta[tid] = tid < len ? beta[(size_t)(t0 + tid) * H + h] : 0.f;

    // ---- P1: cumulative decay and the scaled operands ----
    // thread -> channel pair (c0, c0+1) x sub-tile a1 (rows 16a1..16a1+15).  gam holds
    // the cumsum local to the sub-tile, in log2 units.
    const int c0 = 2 * (tid & 63), a1 = tid >> 6;
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
        *reinterpret_cast<float2 *>(&sm.u.p1.tot[a1][c0]) = run;
        *reinterpret_cast<float2 *>(&sm.u.p1.ref[a1][c0]) = gam[ST / 2 - 1];
    }
    cp_async_wait<0>();
    __syncthreads();
    // pair factors exp(G_ref(a) - G_ref(b)) <= 1 for the off-diagonal sub-tile blocks
#pragma unroll
    for (int m = 0; m < 3; ++m) {
        const int e = tid + 256 * m, p = e >> 7, c = e & (D - 1);
        const int pa = kPairs[p].x, pb = kPairs[p].y;
        float d = sm.u.p1.ref[pa][c] - sm.u.p1.ref[pb][c];
        for (int a = pb; a < pa; ++a) d += sm.u.p1.tot[a][c];
        sm.mfac[p][c] = exp2f(d);
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
        const float2 f1 = make_float2(exp2f(-Gref.x), exp2f(-Gref.y));                   // >= 1
        const float2 f2 = make_float2(exp2f(Gref.x - Gend.x), exp2f(Gref.y - Gend.y));   // >= 1
        const float2 eB = make_float2(exp2f(Ba.x), exp2f(Ba.y));                         // <= 1
        const float2 fC = make_float2(exp2f(GC.x - Ba.x - Gend.x), exp2f(GC.y - Ba.y - Gend.y));
#pragma unroll
        for (int j = 0; j < ST; ++j) {
            const int r = a1 * ST + j;
            const int off = swz128(r, c0);
            // every factor below lies in [e^-80, e^40] for g in (-5, 0]
            const float2 E1 = make_float2(exp2f(gam[j].x), exp2f(gam[j].y));
            const float2 E2 = make_float2(exp2f(Gend.x - gam[j].x), exp2f(Gend.y - gam[j].y));
            const float2 kf = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.r0 + off));
            const float2 qf = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(sm.r1 + off));
            *reinterpret_cast<uint32_t *>(sm.r0 + off) =
                pack_bf16x2(kf.x * E1.x * f1.x, kf.y * E1.y * f1.y);
            *reinterpret_cast<uint32_t *>(sm.r1 + off) =
                pack_bf16x2(qf.x * E1.x * f1.x, qf.y * E1.y * f1.y);
            *reinterpret_cast<uint32_t *>(sm.r3 + off) =
                pack_bf16x2(kf.x * E2.x * f2.x, kf.y * E2.y * f2.y);
            *reinterpret_cast<uint32_t *>(sm.r4 + off) =
                pack_bf16x2(kf.x * E1.x * eB.x, kf.y * E1.y * eB.y);
            *reinterpret_cast<uint32_t *>(rec + REC_QG_SCRATCH + off) =
                pack_bf16x2(qf.x * E1.x * eB.x, qf.y * E1.y * eB.y);
            *reinterpret_cast<uint32_t *>(rec + REC_KT_SCRATCH + off) =
                pack_bf16x2(kf.x * E2.x * fC.x, kf.y * E2.y * fC.y);
        }
        if (a1 == NST - 1)
            *reinterpret_cast<float2 *>(rec + REC_GC + c0 * 4) =
                make_float2(exp2f(GC.x), exp2f(GC.y));
    }
    __syncthreads();

    // ---- P2: key-key and query-key blocks ----
    // warps 0-5: one off-diagonal sub-tile pair each (both products share the
    // rescaled right operand); warps 6-7: two diagonal blocks each, whose
    // key-key blocks they also invert.
    if (warp < 6) {
        const int a = kPairs[warp].x, b = kPairs[warp].y;
        float ak[2][4] = {}, aq[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t lk[4], lq[4], bfr[4];
            ldsm_x4(lk, s0 + swz128(a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
            ldsm_x4(lq, s1 + swz128(a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
            ldsm_x4(bfr, s3 + swz128(b * ST + frag_bn_row(lane), ks * 16 + frag_bn_col(lane)));
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
                *reinterpret_cast<uint32_t *>(sm.aqk + r * LDA + i) =
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
                ldsm_x4(lk, s0 + swz128(a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
                ldsm_x4(lq, s1 + swz128(a * ST + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
                ldsm_x4(bfr, s3 + swz128(a * ST + frag_bn_row(lane), ks * 16 + frag_bn_col(lane)));
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
        {   // lane -> (block a0 + lane/16, column j): solve (I + A_aa) x = e_j in fp32
            const int a = a0 + (lane >> 4), j = lane & 15;
            float x[ST];
#pragma unroll
            for (int r = 0; r < ST; ++r) {
                float sacc = (r == j) ? 1.f : 0.f;
                if (r > j) {
#pragma unroll
                    for (int i = 0; i < r; ++i)
                        if (i >= j) sacc -= sm.u.akd[a][r][i] * x[i];
                }
                x[r] = sacc;
            }
#pragma unroll
            for (int r = 0; r < ST; ++r) sm.taa[a][r * (ST + 8) + j] = f2bf(x[r]);
        }
#pragma unroll
        for (int d = 0; d < 2; ++d)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rl = gid + 8 * hh, il = nt * 8 + 2 * tig;
                    const int r = (a0 + d) * ST + rl, i = (a0 + d) * ST + il;
                    *reinterpret_cast<uint32_t *>(sm.aqk + r * LDA + i) =
                        pack_bf16x2(il <= rl ? aq[d][nt][2 * hh] : 0.f,
                                    il + 1 <= rl ? aq[d][nt][2 * hh + 1] : 0.f);
                }
    }
    __syncthreads();

    // ---- P3: [W|U] = (I + A)^-1 Diag(b) [K*exp G | V] by blocked forward substitution ----
    // warp w owns 32 columns of the solution Y (swz256 over r0..r1): W[:, 32w..] for
    // w < 4, U[:, 32(w-4)..] for w >= 4.  Only warp-level syncs are needed.
    {
        const uint32_t sY = s0;
        uint8_t *Yb = sm.r0;
        __nv_bfloat16 *Z = reinterpret_cast<__nv_bfloat16 *>(sm.r3) + warp * (ST * ZLD);
        const uint8_t *X = warp < 4 ? sm.r4 : sm.r2;
        const int xc = (warp & 3) * 32;   // column base inside X
        const int yc = warp * 32;         // column base inside Y
        for (int a = 0; a < NST; ++a) {
            float acc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = a * ST + gid + 8 * hh;
                    const float2 x = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
                        X + swz128(r, xc + nt * 8 + 2 * tig)));
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
                    ldsm_x4_t(bb, sY + swz256(b * ST + frag_bk_row(lane),
                                              yc + np * 16 + frag_bk_col(lane)));
                    mma_bf16_16816(acc[2 * np], af, bb[0], bb[1]);
                    mma_bf16_16816(acc[2 * np + 1], af, bb[2], bb[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint32_t *>(Z + (gid + 8 * hh) * ZLD + nt * 8 + 2 * tig) =
                        pack_bf16x2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
            __syncwarp();
            float y[4][4] = {};
            uint32_t at[4];
            ldsm_x4(at, smem_u32(sm.taa[a] + frag_a_row(lane) * (ST + 8) + frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bz[4];
                ldsm_x4_t(bz, smem_u32(Z + frag_bk_row(lane) * ZLD + np * 16 + frag_bk_col(lane)));
                mma_bf16_16816(y[2 * np], at, bz[0], bz[1]);
                mma_bf16_16816(y[2 * np + 1], at, bz[2], bz[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = a * ST + gid + 8 * hh;
                    *reinterpret_cast<uint32_t *>(Yb + swz256(r, yc + nt * 8 + 2 * tig)) =
                        pack_bf16x2(y[nt][2 * hh], y[nt][2 * hh + 1]);
                }
            __syncwarp();
        }
    }
    __syncthreads();

    // ---- P4: Kt and Qg back from the record's scratch area into r3 / r4 ----
#pragma unroll
    for (int it = 0; it < 2 * C * D * 2 / 16 / 256; ++it) {
        const int i = tid + it * 256;                  // 16-byte chunk index
        const int m = i / (C * D * 2 / 16), off = (i % (C * D * 2 / 16)) * 16;
        cp_async16((m == 0 ? sm.r3 : sm.r4) + off,
                   rec + (m == 0 ? REC_KT_SCRATCH : REC_QG_SCRATCH) + off);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    // ---- P5: the chunk's affine map ----
    // (a) M' = -Kt^T W and R = Kt^T U: warp w owns key rows 16w..16w+15.
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
        float acc[16][4] = {};
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
            uint32_t ak[4];
            ldsm_x4_t(ak, s3 + swz128(ks * 16 + frag_at_row(lane), warp * 16 + frag_at_col(lane)));
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bb[4];
                ldsm_x4_t(bb, s0 + swz256(ks * 16 + frag_bk_row(lane),
                                          half * D + np * 16 + frag_bk_col(lane)));
                mma_bf16_16816(acc[2 * np], ak, bb[0], bb[1]);
                mma_bf16_16816(acc[2 * np + 1], ak, bb[2], bb[3]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + gid + 8 * hh, c = nt * 8 + 2 * tig;
                if (half == 0)
                    *reinterpret_cast<uint32_t *>(rec + REC_M + swz128(r, c)) =
                        pack_bf16x2(-acc[nt][2 * hh], -acc[nt][2 * hh + 1]);
                else
                    *reinterpret_cast<uint32_t *>(rec + rec_r_off(r, c)) =
                        pack_bf16x2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
            }
    }
    // (b) Q' = Qg - Aqk W and O0 = Aqk U: warp -> chunk rows 16(w&3).., half w>>2.
    {
        const int mt = warp & 3, half = warp >> 2;
        float acc[16][4];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float2 x = make_float2(0.f, 0.f);
                if (half == 0)
                    x = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
                        sm.r4 + swz128(mt * 16 + gid + 8 * hh, nt * 8 + 2 * tig)));
                acc[nt][2 * hh] = -x.x;     // -Qg (negated back on store)
                acc[nt][2 * hh + 1] = -x.y;
            }
        for (int ks = 0; ks <= mt; ++ks) {
            uint32_t aa[4];
            ldsm_x4(aa, smem_u32(sm.aqk + (mt * 16 + frag_a_row(lane)) * LDA + ks * 16 +
                                 frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                uint32_t bb[4];
                ldsm_x4_t(bb, s0 + swz256(ks * 16 + frag_bk_row(lane),
                                          half * D + np * 16 + frag_bk_col(lane)));
                mma_bf16_16816(acc[2 * np], aa, bb[0], bb[1]);
                mma_bf16_16816(acc[2 * np + 1], aa, bb[2], bb[3]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 16; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = mt * 16 + gid + 8 * hh, c = nt * 8 + 2 * tig;
                if (half == 0)
                    *reinterpret_cast<uint32_t *>(rec + REC_QP + swz128(r, c)) =
                        pack_bf16x2(-acc[nt][2 * hh], -acc[nt][2 * hh + 1]);
                else
                    *reinterpret_cast<uint32_t *>(rec + rec_o0_off(r, c)) =
                        pack_bf16x2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
            }
    }
}

// ---------------------------------------------------------------------------
// Kernel 2: inter-chunk state pass.  grid = N * H * (D / DVT), 256 threads.
// Per chunk: S <- Diag(exp G_C) S + M' S + R and O = Q' S + O0, one product
// chain and one barrier.  Warp w owns key rows 16w..16w+15 of the fp32 state
// tile S[:, col0:col0+DVT] (MMA accumulator registers); a double-buffered bf16
// copy in smem is the B operand.  Warps w and w+4 share output rows 16(w&3)..
// and split the tile's columns.  Records arrive by bulk copies into a 3-stage
// mbarrier ring; every wait is bounded (on expiry: timeout bit, drain, return).
// ---------------------------------------------------------------------------
constexpr int NSTAGE = 3;

template <int DVT>
struct StateSmem {
    static constexpr int R_BYTES = D * DVT * 2, O0_BYTES = C * DVT * 2;
    static constexpr int STAGE_BYTES = REC_SHARED + R_BYTES + O0_BYTES;
    uint8_t stage[NSTAGE][STAGE_BYTES];        // [M'|Q'|gC] + R tile + O0 tile
    __nv_bfloat16 sb[2][D * (DVT + 8)];        // bf16 copies of the state tile
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
    using SM = StateSmem<DVT>;
    static_assert(SM::STAGE_BYTES % 128 == 0, "stage alignment");
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SM &sm = *reinterpret_cast<SM *>(smem_raw);
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
        mbar_arrive_expect_tx(bar, SM::STAGE_BYTES);
        if (debug_drop_first_copy && j == 0) return;   // test hook: the wait must run out
        bulk_g2s(dst, rec, REC_SHARED, bar);
        bulk_g2s(dst + REC_SHARED, rec + REC_R + tile * SM::R_BYTES, SM::R_BYTES, bar);
        bulk_g2s(dst + REC_SHARED + SM::R_BYTES, rec + REC_O0 + tile * SM::O0_BYTES,
                 SM::O0_BYTES, bar);
    };
    if (tid == 0)
        for (int j = 0; j < NSTAGE && j < nchunks; ++j) issue(j);

    // state rows 16w..16w+15 -> registers
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
    auto store_sb = [&](int buf) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int r = warp * 16 + gid + 8 * hh;
                *reinterpret_cast<uint32_t *>(sm.sb[buf] + r * LDV + nt * 8 + 2 * tig) =
                    pack_bf16x2(S[nt][2 * hh], S[nt][2 * hh + 1]);
            }
    };
    store_sb(0);
    __syncthreads();

    const int rq = (warp & 3) * 16;       // output rows of this warp
    const int oq = (warp >> 2) * (NT / 2);  // first output n-tile of this warp
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
        const uint32_t sM = smem_u32(st + REC_M), sQ = smem_u32(st + REC_QP);
        const float *gc = reinterpret_cast<const float *>(st + REC_GC);
        const uint8_t *rt = st + REC_SHARED;                 // R tile   [DVT/16][D][16]
        const uint8_t *ot = st + REC_SHARED + SM::R_BYTES;   // O0 tile  [DVT/16][C][16]
        const uint32_t sB = smem_u32(sm.sb[j & 1]);
        const int t0 = seq_t0 + j * C;
        const int len = min(C, seq_len - j * C);

        float acc[NT][4], oacc[NT / 2][4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = warp * 16 + gid + 8 * hh;
            const float gr = gc[r];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int cl = nt * 8 + 2 * tig;
                const float2 rr = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
                    rt + (cl >> 4) * (D * UT * 2) + r * (UT * 2) + (cl & 15) * 2));
                acc[nt][2 * hh] = gr * S[nt][2 * hh] + rr.x;
                acc[nt][2 * hh + 1] = gr * S[nt][2 * hh + 1] + rr.y;
            }
            const int ro = rq + gid + 8 * hh;
#pragma unroll
            for (int i = 0; i < NT / 2; ++i) {
                const int cl = (oq + i) * 8 + 2 * tig;
                const float2 oo = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(
                    ot + (cl >> 4) * (C * UT * 2) + ro * (UT * 2) + (cl & 15) * 2));
                oacc[i][2 * hh] = oo.x;
                oacc[i][2 * hh + 1] = oo.y;
            }
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t am[4], aq[4];
            ldsm_x4(am, sM + swz128(warp * 16 + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
            ldsm_x4(aq, sQ + swz128(rq + frag_a_row(lane), ks * 16 + frag_a_col(lane)));
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b[4];
                ldsm_x4_t(b, sB + 2 * ((ks * 16 + frag_bk_row(lane)) * LDV + np * 16 +
                                       frag_bk_col(lane)));
                mma_bf16_16816(acc[2 * np], am, b[0], b[1]);
                mma_bf16_16816(acc[2 * np + 1], am, b[2], b[3]);
                if constexpr (NT == 2) {
                    if (oq == 0) mma_bf16_16816(oacc[0], aq, b[0], b[1]);
                    else mma_bf16_16816(oacc[0], aq, b[2], b[3]);
                } else {
                    if (2 * np == oq) {
                        mma_bf16_16816(oacc[0], aq, b[0], b[1]);
                        mma_bf16_16816(oacc[1], aq, b[2], b[3]);
                    }
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) S[nt][e] = acc[nt][e];
        store_sb((j + 1) & 1);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int r = rq + gid + 8 * hh;
            if (r < len) {
                __nv_bfloat16 *orow = o + ((size_t)(t0 + r) * H + h) * D + col0;
#pragma unroll
                for (int i = 0; i < NT / 2; ++i)
                    *reinterpret_cast<uint32_t *>(orow + (oq + i) * 8 + 2 * tig) =
                        pack_bf16x2(oacc[i][2 * hh], oacc[i][2 * hh + 1]);
            }
        }
        __syncthreads();   // new state copy ready; stage s consumed
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
