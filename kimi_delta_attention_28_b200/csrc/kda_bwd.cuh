// kda_bwd.cuh -- gradient of the KDA recurrence (backward pass), fp32 on CUDA cores.
//
// The recurrence ("Kimi K3" open-weights field notes, panel "KDA 单头递归"), per
// token with S' = Diag(exp g) S_{t-1}, u = S'^T k, delta = v - u:
//     S_t = S' + beta k delta^T,   o_t = S_t^T q.
// Given dO = dL/do and dhT = dL/dS_T, the chain rule from the last token to the
// first, with G = dL/dS_t:
//     G += q do^T;  dq = S_t do;  w = G delta;  dbeta = k . w;
//     dd = beta G^T k (= dv);  dk = beta w - S' dd;
//     G' = G - k dd^T;  dg_i = sum_j S'_ij G'_ij;  G = Diag(exp g) G';   dh0 = G.
// The state's value columns evolve independently in both directions (the forward
// update and the G update act column by column), so a CTA owns one 32-column slice
// of one (sequence, head) chain.  It runs the chain forward once, storing its slice
// of the state every CK tokens in HBM; then it walks the CK-token chunks backwards:
// from a chunk's checkpoint it recomputes the state every CB tokens into a small
// scratch of its own (L2-resident), and for each CB-token piece, last first, the
// piece's states into shared memory, to which it applies the rules above.  dv and
// dh0 columns are complete within a slice; dq, dk, dg and dbeta are sums over all
// columns: the D/16 slice CTAs of a chain form a thread-block cluster, and after
// every piece each CTA adds the slices' partial sums for D/(D/16) of the rows
// through distributed shared memory, in slice order (deterministic).
// Segments: with nseg > 1 (fixed-length input) a chain is cut into nseg segments of
// seg_chunks chunks, one cluster each, all running at once.  A segment starts from the
// state at its first token (h0 for the first segment, else s_start) and its reverse
// pass from dL/dS at its last token (dL/dhT for the last segment, else g_end); both
// come from the tensor-core forward and the chunk-level gradient chain
// (kda_bwd_chain.cuh), whose checkpoints every seg_chunks chunks they are.
// Inside a CTA, warp w owns 4 columns of the slice across all d rows (lane l: rows
// RPL l .. RPL l + RPL - 1, RPL = d / 32), so the column sums every token needs
// (u = S'^T k, G^T k) are in-warp butterflies with no CTA barrier; the row sums
// (dq, dk, dg, dbeta) are only outputs, so each warp's share goes to shared memory
// and the four shares are added once per token.  (Keeping every token's shares of a
// piece and adding them once per piece needs 37 KiB more shared memory, one CTA per
// SM instead of two, and the 8-CTA clusters then no longer fit the GPU at once.)
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int SLC = 16;   // value columns per CTA
constexpr int CK = 64;    // tokens per stored checkpoint (HBM)
constexpr int CB = 8;     // tokens per recompute piece (their states live in smem)
constexpr int NSUB = CK / CB;

template <typename TIn>
KDA_DEVINL float ldf(const TIn *p);
template <>
KDA_DEVINL float ldf<float>(const float *p) { return __ldg(p); }
template <>
KDA_DEVINL float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) { return bf2f(*p); }
KDA_DEVINL float to_f(float x) { return x; }
KDA_DEVINL float to_f(__nv_bfloat16 x) { return bf2f(x); }
template <typename TIn>
KDA_DEVINL void stf(TIn *p, float x);
template <>
KDA_DEVINL void stf<float>(float *p, float x) { *p = x; }
template <>
KDA_DEVINL void stf<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = f2bf(x); }

// Checkpoint slot of chunk j of a sequence starting at token t0 of the flattened
// token axis, sequence index n: floor(t0 / CK) + n + j.  Distinct sequences get
// disjoint slot ranges, and slots < T_total / CK + N + 1.
KDA_DEVINL long long ckpt_slot(int t0, int n, int j) { return (long long)(t0 / CK) + n + j; }

// Distributed shared memory: the shared-memory address of `p` in CTA `rank` of the
// cluster, and a load from it.
KDA_DEVINL uint32_t dsmem_addr(const void *p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}
// (No memory clobber: a run of these loads may be issued back to back; the cluster
// barriers around them, which do clobber memory, keep them in place.)
KDA_DEVINL float dsmem_ld(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr));
    return v;
}
KDA_DEVINL void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

constexpr int NWB = SLC / 4;   // warps per CTA (4 columns each)
constexpr int NTB = 32 * NWB;   // threads per CTA

// Row-sum slots of one token (dq, dk, dg rows, then dbeta), padded to 16 bytes.
template <int D>
constexpr int psw() { return 3 * D + 4; }

// RPL consecutive fp32 values from shared memory (16-byte aligned for RPL = 4), as
// one vector access.
template <int RPL>
KDA_DEVINL void ld_rows(const float *p, float (&x)[RPL]) {
    if constexpr (RPL == 4) {
        const float4 v = *reinterpret_cast<const float4 *>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else if constexpr (RPL == 2) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        x[0] = v.x; x[1] = v.y;
    } else {
        x[0] = *p;
    }
}
template <int RPL>
KDA_DEVINL void st_rows(float *p, const float (&x)[RPL]) {
    if constexpr (RPL == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (RPL == 2) {
        *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
    } else {
        *p = x[0];
    }
}

template <int D, typename TIn>
struct BwdSmem {
    // states S_{t-1} of the piece's tokens: each thread's own RPL x 4 block, stored
    // thread-minor (the 16-byte vectors of consecutive threads are adjacent, so a warp's
    // access is conflict-free; the data never leaves the thread that wrote it)
    float4 st[CB][D / 32][NTB];
    float q[CB][D], k[CB][D], a[CB][D];   // a = exp(g)
    float v[CB][SLC], dO[CB][SLC];
    float b[CB];
    float pw[2][NWB][psw<D>()];   // each warp's share of a token's dq, dk, dg, dbeta
    float ps[CB][psw<D>()];       // this slice's partial dq, dk, dg rows and dbeta per token
    // the next piece's inputs as they arrive (asynchronous copies, input dtype)
    __align__(16) TIn xk[CB][D];
    __align__(16) TIn xq[CB][D];
    __align__(16) float xg[CB][D];
    __align__(16) TIn xv[CB][SLC];
    __align__(16) TIn xdo[CB][SLC];
    __align__(16) float xb[CB];
};

// Sum of x over the 32 lanes of the warp, left in every lane.
KDA_DEVINL float warp_sum(float x) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NTB, 1)
kda_bwd_slice_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                     const TIn *__restrict__ v, const float *__restrict__ g,
                     const float *__restrict__ beta, const float *__restrict__ h0,
                     const int *__restrict__ cu, const int *__restrict__ hdr,
                     const TIn *__restrict__ dO, const float *__restrict__ dhT, int T, int H,
                     float *__restrict__ ckpt, float *__restrict__ sub, TIn *__restrict__ dq,
                     TIn *__restrict__ dk, TIn *__restrict__ dv, float *__restrict__ dg,
                     float *__restrict__ dbeta, float *__restrict__ dh0, long long ntok,
                     int *err_word, int nseg, int seg_chunks, const float *__restrict__ s_start,
                     const float *__restrict__ g_end, int nfw, int cps) {
    constexpr int NS = D / SLC, NT = NTB, RPL = D / 32;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BwdSmem<D, TIn> &sm = *reinterpret_cast<BwdSmem<D, TIn> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r0 = RPL * lane, c4 = 4 * warp;        // this thread: rows r0.., slice columns c4..
    const int slice = blockIdx.x % NS, unit = blockIdx.x / NS;
    const int chain = unit / nseg, seg = unit % nseg, n = chain / H, h = chain % H;
    const int cs = slice * SLC;                      // the slice's first column
    int t0, len;
    if (cu) {
        if (!hdr[0]) return;
        t0 = cu[n];
        len = cu[n + 1] - cu[n];
    } else {
        t0 = n * T;
        len = T;
    }
    if (nseg > 1) {   // this unit's tokens: seg_chunks chunks from the segment's start
        const int lo = seg * seg_chunks * CK;
        t0 += lo;
        len = min(len - lo, seg_chunks * CK);
    }
    if constexpr (KDA_DEBUG) {
        if (len < 0 || t0 < 0 || (long long)t0 + len > ntok) {
            if (tid == 0) atomicOr(err_word, kErrBoundsBit);
            return;
        }
    }
    const int nck = (len + CK - 1) / CK;
    // this thread's RPL x 4 block of a [D][D] state (h0, dhT, dh0, checkpoints) and of
    // the CTA's [D][SLC] scratch
    const size_t sbase = (size_t)chain * D * D + cs + c4;
    float *mysub = sub + (size_t)blockIdx.x * NSUB * D * SLC + c4;
    auto ldS = [&](float (&S)[RPL][4], const float *base, int ld) {
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const float4 x = *reinterpret_cast<const float4 *>(base + (size_t)(r0 + i) * ld);
            S[i][0] = x.x; S[i][1] = x.y; S[i][2] = x.z; S[i][3] = x.w;
        }
    };
    auto stS = [&](float *base, int ld, const float (&S)[RPL][4]) {
#pragma unroll
        for (int i = 0; i < RPL; ++i)
            *reinterpret_cast<float4 *>(base + (size_t)(r0 + i) * ld) =
                make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
    };
    // A piece's inputs in shared memory (tokens p0 .. p0 + cl - 1 of the sequence): q,
    // k, exp(g) rows; this slice's v, dO columns; beta.  They arrive one piece ahead by
    // asynchronous copies (rows past the piece zero-filled) into a staging area: when
    // a piece is due, its copies are awaited, converted to fp32 in place for the
    // steps, and the copies of the next piece in the kernel's order are issued, so
    // their latency hides behind the current piece's work (CTA barriers do not wait
    // for them).  The order: the forward walk's pieces (phase 1, chunks 0 .. nck - 2),
    // then per chunk from the last, its recompute walk (phase 2, pieces 0 .. npc - 2)
    // and its backward pieces (phase 3, npc - 1 .. 0, which also need q and dO).
    struct Ev {
        int ph, j, pc;   // ph 0: none
    };
    auto npc_of = [&](int j) { return (min(CK, len - j * CK) + CB - 1) / CB; };
    auto first_back = [&](int j) -> Ev {
        const int npc = npc_of(j);
        return npc >= 2 ? Ev{2, j, 0} : Ev{3, j, npc - 1};
    };
    auto next_ev = [&](Ev e) -> Ev {
        if (e.ph == 1) {
            if (e.pc + 1 < npc_of(e.j)) return Ev{1, e.j, e.pc + 1};
            if (e.j + 2 < nck) return Ev{1, e.j + 1, 0};
            return first_back(nck - 1);
        }
        if (e.ph == 2) {
            if (e.pc + 1 <= npc_of(e.j) - 2) return Ev{2, e.j, e.pc + 1};
            return Ev{3, e.j, npc_of(e.j) - 1};
        }
        if (e.ph == 3) {
            if (e.pc > 0) return Ev{3, e.j, e.pc - 1};
            if (e.j > 0) return first_back(e.j - 1);
        }
        return Ev{0, 0, 0};
    };
    auto issue_stage = [&](Ev e) {
        if (e.ph == 0) return;
        const int p0 = e.j * CK + e.pc * CB, cl = min(CB, len - p0), c0 = t0 + p0;
        const bool with_q = e.ph == 3;
        constexpr int RC = D * (int)sizeof(TIn) / 16;   // 16-byte pieces of a q / k row
        constexpr int GC = D * 4 / 16;                   // ... of a g row
        constexpr int VC = SLC * (int)sizeof(TIn) / 16;  // ... of the slice of a v / dO row
        for (int x = tid; x < CB * RC; x += NT) {
            const int i = x / RC, ch = x % RC, ii = min(i, cl - 1);   // a valid source row
            const size_t row = ((size_t)(c0 + ii) * H + h) * D;
            const int nb = i < cl ? 16 : 0;
            cp_async16(reinterpret_cast<uint8_t *>(sm.xk[i]) + 16 * ch,
                       reinterpret_cast<const uint8_t *>(k + row) + 16 * ch, nb);
            if (with_q)
                cp_async16(reinterpret_cast<uint8_t *>(sm.xq[i]) + 16 * ch,
                           reinterpret_cast<const uint8_t *>(q + row) + 16 * ch, nb);
        }
        for (int x = tid; x < CB * GC; x += NT) {
            const int i = x / GC, ch = x % GC, ii = min(i, cl - 1);
            cp_async16(reinterpret_cast<uint8_t *>(sm.xg[i]) + 16 * ch,
                       reinterpret_cast<const uint8_t *>(g + ((size_t)(c0 + ii) * H + h) * D) +
                           16 * ch,
                       i < cl ? 16 : 0);
        }
        for (int x = tid; x < CB * VC; x += NT) {
            const int i = x / VC, ch = x % VC, ii = min(i, cl - 1);
            const size_t row = ((size_t)(c0 + ii) * H + h) * D + cs;
            const int nb = i < cl ? 16 : 0;
            cp_async16(reinterpret_cast<uint8_t *>(sm.xv[i]) + 16 * ch,
                       reinterpret_cast<const uint8_t *>(v + row) + 16 * ch, nb);
            if (with_q)
                cp_async16(reinterpret_cast<uint8_t *>(sm.xdo[i]) + 16 * ch,
                           reinterpret_cast<const uint8_t *>(dO + row) + 16 * ch, nb);
        }
        if (tid < CB)
            cp_async4(&sm.xb[tid], beta + (size_t)(c0 + min(tid, cl - 1)) * H + h, tid < cl ? 4 : 0);
        cp_async_commit();
    };
    Ev cur = nck > 1 ? Ev{1, 0, 0} : (nck == 1 ? first_back(0) : Ev{0, 0, 0});
    issue_stage(cur);
    auto stage = [&]() {
        const bool with_q = cur.ph == 3;
        cp_async_wait<0>();
        __syncthreads();   // every thread's copies of the piece have landed
        for (int e = tid; e < CB * D; e += NT) {
            const int i = e / D, c = e % D;
            sm.k[i][c] = to_f(sm.xk[i][c]);
            sm.a[i][c] = expf(sm.xg[i][c]);   // exp(0) = 1 past the piece
            if (with_q) sm.q[i][c] = to_f(sm.xq[i][c]);
        }
        for (int e = tid; e < CB * SLC; e += NT) {
            const int i = e / SLC, c = e % SLC;
            sm.v[i][c] = to_f(sm.xv[i][c]);
            if (with_q) sm.dO[i][c] = to_f(sm.xdo[i][c]);
        }
        if (tid < CB) sm.b[tid] = sm.xb[tid];
        __syncthreads();   // converted; the staging area is free for the next piece
        cur = next_ev(cur);
        issue_stage(cur);
    };
    // one token of the recurrence on this thread's block; returns delta = v - u for the
    // warp's 4 columns (the same in every lane)
    auto step = [&](float (&S)[RPL][4], int i, float (&dl)[4]) {
        float u[4] = {0.f, 0.f, 0.f, 0.f}, av[RPL], kv[RPL];
        ld_rows<RPL>(&sm.a[i][r0], av);
        ld_rows<RPL>(&sm.k[i][r0], kv);
#pragma unroll
        for (int ri = 0; ri < RPL; ++ri) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                S[ri][c] *= av[ri];
                u[c] = fmaf(kv[ri], S[ri][c], u[c]);
            }
        }
        const float b = sm.b[i];
        const float4 vv = *reinterpret_cast<const float4 *>(&sm.v[i][c4]);
        dl[0] = vv.x - warp_sum(u[0]);
        dl[1] = vv.y - warp_sum(u[1]);
        dl[2] = vv.z - warp_sum(u[2]);
        dl[3] = vv.w - warp_sum(u[3]);
#pragma unroll
        for (int ri = 0; ri < RPL; ++ri) {
            const float bk = b * kv[ri];
#pragma unroll
            for (int c = 0; c < 4; ++c) S[ri][c] = fmaf(bk, dl[c], S[ri][c]);
        }
    };
    // run the tokens p0 .. p0 + cl - 1 forward from S (inputs staged here)
    auto run = [&](float (&S)[RPL][4], int p0, int cl) {
        (void)p0;   // staged in order (see stage)
        stage();
        float dl[4];
        for (int i = 0; i < cl; ++i) step(S, i, dl);
        __syncthreads();   // the next staging overwrites the inputs
    };

    // ---- forward: the slice's state at the start of every CK-token chunk, to HBM ----
    // (the state after the last chunk is not needed: the walk stops before it)
    float S[RPL][4];
    const float *s_init = seg == 0 ? (h0 ? h0 + sbase : nullptr)
                                   : s_start + ((size_t)(n * nfw + seg - 1) * H + h) * D * D + cs + c4;
    if (s_init) ldS(S, s_init, D);
    else
#pragma unroll
        for (int i = 0; i < RPL; ++i) S[i][0] = S[i][1] = S[i][2] = S[i][3] = 0.f;
    for (int j = 0; j < nck; ++j) {
        stS(ckpt + (ckpt_slot(t0, n, j) * H + h) * D * D + cs + c4, D, S);
        const int lenj = min(CK, len - j * CK);
        if (j + 1 < nck)
            for (int p = 0; p < lenj; p += CB) run(S, j * CK + p, min(CB, lenj - p));
    }

    // ---- backward ----
    // dL/dS after the unit's last token: dL/dhT, or the chain's checkpoint at the
    // boundary (seg + 1) seg_chunks chunks, which it stored after cps - (seg + 1)
    // seg_chunks of its (reversed) steps
    float G[RPL][4];
    const float *g_init = seg == nseg - 1
                              ? (dhT ? dhT + sbase : nullptr)
                              : g_end + ((size_t)(n * nfw + cps / seg_chunks - seg - 2) * H + h) * D * D + cs + c4;
    if (g_init) ldS(G, g_init, D);
    else
#pragma unroll
        for (int i = 0; i < RPL; ++i) G[i][0] = G[i][1] = G[i][2] = G[i][3] = 0.f;
    const uint32_t cl_rank = (uint32_t)slice;   // the cluster holds the chain's NS slices
    int tok = 0;                                // tokens done: parity of the pw buffer
    for (int j = nck - 1; j >= 0; --j) {
        const int lenj = min(CK, len - j * CK), npc = (lenj + CB - 1) / CB;
        // the state every CB tokens of the chunk, from its checkpoint, to this CTA's scratch
        ldS(S, ckpt + (ckpt_slot(t0, n, j) * H + h) * D * D + cs + c4, D);
        for (int pc = 0; pc < npc; ++pc) {
            stS(mysub + (size_t)pc * D * SLC, SLC, S);
            if (pc + 1 < npc) run(S, j * CK + pc * CB, min(CB, lenj - pc * CB));
        }
        for (int pc = npc - 1; pc >= 0; --pc) {
            const int p0 = j * CK + pc * CB, cl = min(CB, lenj - pc * CB);
            stage();
            ldS(S, mysub + (size_t)pc * D * SLC, SLC);
            float dls[CB][4];   // delta of every token of the piece (this warp's columns)
#pragma unroll
            for (int i = 0; i < CB; ++i) {   // recompute: S_{t-1} of every token to smem
                if (i < cl) {
#pragma unroll
                    for (int ri = 0; ri < RPL; ++ri)
                        sm.st[i][ri][tid] = make_float4(S[ri][0], S[ri][1], S[ri][2], S[ri][3]);
                    step(S, i, dls[i]);
                }
            }
#pragma unroll
            for (int i = CB - 1; i >= 0; --i) {
                if (i >= cl) continue;
                const float b = sm.b[i];
                float Sp[RPL][4], dov[4], av[RPL], kv[RPL], qv[RPL];
                {
                    const float4 d4 = *reinterpret_cast<const float4 *>(&sm.dO[i][c4]);
                    dov[0] = d4.x; dov[1] = d4.y; dov[2] = d4.z; dov[3] = d4.w;
                }
                ld_rows<RPL>(&sm.a[i][r0], av);
                ld_rows<RPL>(&sm.k[i][r0], kv);
                ld_rows<RPL>(&sm.q[i][r0], qv);
                // G += q do^T; dq = S_t do with S_t = S' + b k delta^T; w = G delta
                float pq[RPL], pwr[RPL], xk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ri = 0; ri < RPL; ++ri) {
                    const float a = av[ri], kr = kv[ri], qr = qv[ri];
                    const float4 sv = sm.st[i][ri][tid];
                    Sp[ri][0] = a * sv.x; Sp[ri][1] = a * sv.y; Sp[ri][2] = a * sv.z; Sp[ri][3] = a * sv.w;
                    pq[ri] = 0.f;
                    pwr[ri] = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        G[ri][c] = fmaf(qr, dov[c], G[ri][c]);
                        pq[ri] = fmaf(fmaf(b * kr, dls[i][c], Sp[ri][c]), dov[c], pq[ri]);
                        pwr[ri] = fmaf(G[ri][c], dls[i][c], pwr[ri]);
                        xk[c] = fmaf(kr, G[ri][c], xk[c]);
                    }
                }
                // dd = b G^T k for the warp's columns (complete: this CTA owns them)
                float dd[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) dd[c] = b * warp_sum(xk[c]);
                if (lane < 4)
                    stf<TIn>(dv + ((size_t)(t0 + p0 + i) * H + h) * D + cs + c4 + lane,
                             lane == 0 ? dd[0] : lane == 1 ? dd[1] : lane == 2 ? dd[2] : dd[3]);
                float pbeta = 0.f, pk[RPL], pgs[RPL];
                float *pwb = sm.pw[tok & 1][warp];
#pragma unroll
                for (int ri = 0; ri < RPL; ++ri) {
                    const float a = av[ri], kr = kv[ri];
                    float px = 0.f, pg = 0.f;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        px = fmaf(Sp[ri][c], dd[c], px);
                        const float gp = G[ri][c] - kr * dd[c];
                        pg = fmaf(Sp[ri][c], gp, pg);
                        G[ri][c] = a * gp;
                    }
                    pk[ri] = b * pwr[ri] - px;
                    pgs[ri] = pg;
                    pbeta = fmaf(kr, pwr[ri], pbeta);
                }
                st_rows<RPL>(pwb + r0, pq);
                st_rows<RPL>(pwb + D + r0, pk);
                st_rows<RPL>(pwb + 2 * D + r0, pgs);
                pbeta = warp_sum(pbeta);
                if (lane == 0) pwb[3 * D] = pbeta;
                __syncthreads();
                // the warps' shares, added in warp order, into the piece's partial sums
                for (int e = tid; e < 3 * D + 1; e += NT) {
                    float sum = 0.f;
#pragma unroll
                    for (int w = 0; w < NWB; ++w) sum += sm.pw[tok & 1][w][e];
                    sm.ps[i][e] = sum;
                }
                ++tok;
            }
            // the slices' partial sums of the piece: every CTA of the cluster adds them for
            // D / NS rows (and CTA 0 for dbeta), in slice order
            cluster_sync();
            {
                constexpr int RPC = D / NS;                   // rows per CTA
                for (int e = tid; e < cl * (3 * RPC + 1); e += NT) {
                    const int i = e / (3 * RPC + 1), f = e % (3 * RPC + 1);
                    if (f == 3 * RPC && cl_rank != 0) continue;
                    const int col = f == 3 * RPC ? 3 * D : (f / RPC) * D + cl_rank * RPC + f % RPC;
                    float part[NS];   // all the slices' loads in flight at once, then added in order
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) part[sl] = dsmem_ld(dsmem_addr(&sm.ps[i][col], sl));
                    float sum = 0.f;
#pragma unroll
                    for (int sl = 0; sl < NS; ++sl) sum += part[sl];
                    const size_t u = (size_t)(t0 + p0 + i) * H + h;
                    if (f == 3 * RPC) {
                        dbeta[u] = sum;
                    } else {
                        const int kind = f / RPC, row = cl_rank * RPC + f % RPC;
                        if (kind == 0) stf<TIn>(dq + u * D + row, sum);
                        else if (kind == 1) stf<TIn>(dk + u * D + row, sum);
                        else dg[u * D + row] = sum;
                    }
                }
            }
            cluster_sync();   // the partial sums may be overwritten by the next piece
        }
    }
    if (dh0 && seg == 0) stS(dh0 + sbase, D, G);
}

}  // namespace bwd
}  // namespace kda
