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
// of one (sequence, head) chain: it runs the chain forward once, storing its slice
// of the state every CB tokens, then walks the chunks of CB tokens backwards,
// recomputing each chunk's states into shared memory and applying the rules above.
// dv and dh0 columns are complete within a slice; dq, dk, dg and dbeta are sums over
// all columns, so every slice writes its partial sums and a second kernel adds the
// slices (in a fixed order: the result does not depend on scheduling).
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int SLC = 32;   // value columns per CTA
constexpr int CB = 8;     // tokens per recompute chunk (states of a chunk live in smem)

template <typename TIn>
KDA_DEVINL float ldf(const TIn *p);
template <>
KDA_DEVINL float ldf<float>(const float *p) { return __ldg(p); }
template <>
KDA_DEVINL float ldf<__nv_bfloat16>(const __nv_bfloat16 *p) { return bf2f(*p); }
template <typename TIn>
KDA_DEVINL void stf(TIn *p, float x);
template <>
KDA_DEVINL void stf<float>(float *p, float x) { *p = x; }
template <>
KDA_DEVINL void stf<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = f2bf(x); }

// Checkpoint slot of chunk j of a sequence starting at token t0 of the flattened
// token axis, sequence index n: floor(t0 / CB) + n + j.  Distinct sequences get
// disjoint slot ranges, and slots < T_total / CB + N + 1.
KDA_DEVINL long long ckpt_slot(int t0, int n, int j) { return (long long)(t0 / CB) + n + j; }

template <int D>
struct BwdSmem {
    float st[CB][D][SLC];      // states S_{t-1} of the chunk's tokens (this slice)
    float q[CB][D], k[CB][D], a[CB][D];   // a = exp(g)
    float v[CB][SLC], dO[CB][SLC], delta[CB][SLC];
    float b[CB];
    float part[D / 16][SLC];   // column-reduction partials, one row per warp
    float vec[SLC];            // column-reduction result
    float red[D / 16];         // dbeta partials, one per warp
};

// Column sum over the D rows of x (thread: row tid/2, columns 16 (tid & 1) .. +15 of
// the slice).  Within a warp (16 rows x 2 column halves) a reduce-scatter over the
// four row bits of the lane leaves lane l with one column summed over the warp's
// rows; the warps' partials are added through shared memory.  The result for this
// thread's 16 columns is returned in out; the CTA synchronises twice.
template <int D>
KDA_DEVINL void col_sum(BwdSmem<D> &sm, const float (&x)[16], float (&out)[16]) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ch = tid & 1;
    float c8[8], c4[4], c2[2];
    {
        const bool up = lane & 2;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float send = up ? x[p] : x[p + 8];
            c8[p] = (up ? x[p + 8] : x[p]) + __shfl_xor_sync(0xffffffffu, send, 2);
        }
    }
    {
        const bool up = lane & 4;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const float send = up ? c8[p] : c8[p + 4];
            c4[p] = (up ? c8[p + 4] : c8[p]) + __shfl_xor_sync(0xffffffffu, send, 4);
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const float send = up ? c4[p] : c4[p + 2];
            c2[p] = (up ? c4[p + 2] : c4[p]) + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    float c1;
    {
        const bool up = lane & 16;
        const float send = up ? c2[0] : c2[1];
        c1 = (up ? c2[1] : c2[0]) + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    // lane bits 1..4 chose the halves 8, 4, 2, 1: the column within this half
    const int col = ((lane >> 1) & 1) * 8 + ((lane >> 2) & 1) * 4 + ((lane >> 3) & 1) * 2 +
                    ((lane >> 4) & 1);
    sm.part[warp][ch * 16 + col] = c1;
    __syncthreads();
    if (tid < SLC) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < D / 16; ++w) s += sm.part[w][tid];
        sm.vec[tid] = s;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 16; c += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(&sm.vec[ch * 16 + c]);
        out[c] = t.x;
        out[c + 1] = t.y;
        out[c + 2] = t.z;
        out[c + 3] = t.w;
    }
}

template <int D, typename TIn>
__global__ void __launch_bounds__(2 * D, 1)
kda_bwd_slice_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                     const TIn *__restrict__ v, const float *__restrict__ g,
                     const float *__restrict__ beta, const float *__restrict__ h0,
                     const int *__restrict__ cu, const int *__restrict__ hdr,
                     const TIn *__restrict__ dO, const float *__restrict__ dhT, int T, int H,
                     float *__restrict__ ckpt, float *__restrict__ part, TIn *__restrict__ dv,
                     float *__restrict__ dh0, long long ntok, int *err_word) {
    constexpr int NS = D / SLC, NT = 2 * D;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BwdSmem<D> &sm = *reinterpret_cast<BwdSmem<D> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int r = tid >> 1, ch = tid & 1;
    const int slice = blockIdx.x % NS, chain = blockIdx.x / NS, n = chain / H, h = chain % H;
    const int cs = slice * SLC, cc = cs + ch * 16;   // slice's first column, this thread's
    int t0, len;
    if (cu) {
        if (!hdr[0]) return;
        t0 = cu[n];
        len = cu[n + 1] - cu[n];
    } else {
        t0 = n * T;
        len = T;
    }
    if constexpr (KDA_DEBUG) {
        if (len < 0 || t0 < 0 || (long long)t0 + len > ntok) {
            if (tid == 0) atomicOr(err_word, kErrBoundsBit);
            return;
        }
    }
    const int nch = (len + CB - 1) / CB;
    const size_t sstate = (size_t)chain * D * D + (size_t)r * D + cc;   // h0 / dhT / dh0 offset
    // a chunk's inputs into shared memory: q, k, exp(g) rows; this slice's v, dO columns
    auto stage = [&](int j, bool with_q) {
        const int c0 = t0 + j * CB, cl = min(CB, len - j * CB);
        for (int e = tid; e < CB * D; e += NT) {
            const int i = e / D, c = e % D;
            const bool in = i < cl;
            const size_t row = ((size_t)(c0 + i) * H + h) * D + c;
            sm.k[i][c] = in ? ldf<TIn>(k + row) : 0.f;
            sm.a[i][c] = in ? expf(__ldg(g + row)) : 1.f;
            if (with_q) sm.q[i][c] = in ? ldf<TIn>(q + row) : 0.f;
        }
        for (int e = tid; e < CB * SLC; e += NT) {
            const int i = e / SLC, c = e % SLC;
            const bool in = i < cl;
            const size_t row = ((size_t)(c0 + i) * H + h) * D + cs + c;
            sm.v[i][c] = in ? ldf<TIn>(v + row) : 0.f;
            if (with_q) sm.dO[i][c] = in ? ldf<TIn>(dO + row) : 0.f;
        }
        if (tid < CB) sm.b[tid] = tid < cl ? __ldg(beta + (size_t)(c0 + tid) * H + h) : 0.f;
        __syncthreads();
    };
    // one token of the recurrence on this thread's part of the state; delta to smem
    auto step = [&](float (&S)[16], int i, bool keep_delta) {
        const float a = sm.a[i][r], kr = sm.k[i][r], b = sm.b[i];
        float x[16], u[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            S[c] *= a;
            x[c] = kr * S[c];
        }
        col_sum<D>(sm, x, u);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float dl = sm.v[i][ch * 16 + c] - u[c];
            S[c] = fmaf(b * kr, dl, S[c]);
            if (keep_delta && r == 0) sm.delta[i][ch * 16 + c] = dl;
        }
    };

    // ---- forward: the slice's state at the start of every chunk ----
    float S[16];
#pragma unroll
    for (int c = 0; c < 16; c += 4) {
        const float4 x = h0 ? *reinterpret_cast<const float4 *>(h0 + sstate + c)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        S[c] = x.x; S[c + 1] = x.y; S[c + 2] = x.z; S[c + 3] = x.w;
    }
    for (int j = 0; j < nch; ++j) {
        float *cp = ckpt + ((ckpt_slot(t0, n, j) * H + h) * D + r) * D + cc;
#pragma unroll
        for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4 *>(cp + c) = make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
        stage(j, false);
        const int cl = min(CB, len - j * CB);
        for (int i = 0; i < cl; ++i) step(S, i, false);
        __syncthreads();   // the next chunk's staging overwrites the inputs
    }

    // ---- backward ----
    float G[16];
#pragma unroll
    for (int c = 0; c < 16; c += 4) {
        const float4 x = dhT ? *reinterpret_cast<const float4 *>(dhT + sstate + c)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        G[c] = x.x; G[c + 1] = x.y; G[c + 2] = x.z; G[c + 3] = x.w;
    }
    const size_t pstride = (size_t)ntok * H;   // partial sums: [NS][ntok * H][3 D + 1]
    for (int j = nch - 1; j >= 0; --j) {
        const int cl = min(CB, len - j * CB);
        stage(j, true);
        const float *cp = ckpt + ((ckpt_slot(t0, n, j) * H + h) * D + r) * D + cc;
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(cp + c);
            S[c] = x.x; S[c + 1] = x.y; S[c + 2] = x.z; S[c + 3] = x.w;
        }
        for (int i = 0; i < cl; ++i) {   // recompute: S_{t-1} of every token to smem
#pragma unroll
            for (int c = 0; c < 16; c += 4)
                *reinterpret_cast<float4 *>(&sm.st[i][r][ch * 16 + c]) =
                    make_float4(S[c], S[c + 1], S[c + 2], S[c + 3]);
            step(S, i, true);
        }
        __syncthreads();   // delta visible
        for (int i = cl - 1; i >= 0; --i) {
            const int t = t0 + j * CB + i;
            const float a = sm.a[i][r], kr = sm.k[i][r], qr = sm.q[i][r], b = sm.b[i];
            float Sp[16], dl[16], dov[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                Sp[c] = a * sm.st[i][r][ch * 16 + c];
                dl[c] = sm.delta[i][ch * 16 + c];
                dov[c] = sm.dO[i][ch * 16 + c];
            }
            // G += q do^T; dq = S_t do with S_t = S' + b k delta^T; w = G delta
            float pq = 0.f, pw = 0.f, x[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                G[c] = fmaf(qr, dov[c], G[c]);
                pq = fmaf(fmaf(b * kr, dl[c], Sp[c]), dov[c], pq);
                pw = fmaf(G[c], dl[c], pw);
                x[c] = kr * G[c];
            }
            pq += __shfl_xor_sync(0xffffffffu, pq, 1);
            pw += __shfl_xor_sync(0xffffffffu, pw, 1);
            // dd = b G^T k: the column sum (complete: this CTA owns the columns)
            float dd[16];
            col_sum<D>(sm, x, dd);
            if (tid < SLC) stf<TIn>(dv + ((size_t)t * H + h) * D + cs + tid, b * sm.vec[tid]);
            float px = 0.f, pg = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                dd[c] *= b;
                px = fmaf(Sp[c], dd[c], px);
                const float gp = G[c] - kr * dd[c];
                pg = fmaf(Sp[c], gp, pg);
                G[c] = a * gp;
            }
            px += __shfl_xor_sync(0xffffffffu, px, 1);
            pg += __shfl_xor_sync(0xffffffffu, pg, 1);
            // dbeta partial = sum over rows of k_r w_r (rows of this warp, then warps)
            float pb = ch == 0 ? kr * pw : 0.f;
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) pb += __shfl_xor_sync(0xffffffffu, pb, m);
            if (lane == 0) sm.red[warp] = pb;
            float *pp = part + ((size_t)slice * pstride + (size_t)t * H + h) * (3 * D + 1);
            if (ch == 0) {
                pp[r] = pq;
                pp[D + r] = b * pw - px;
                pp[2 * D + r] = pg;
            }
            __syncthreads();
            if (tid == 0) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < D / 16; ++w) s += sm.red[w];
                pp[3 * D] = s;
            }
        }
        __syncthreads();   // the next chunk's staging overwrites the inputs and states
    }
    if (dh0) {
#pragma unroll
        for (int c = 0; c < 16; c += 4)
            *reinterpret_cast<float4 *>(dh0 + sstate + c) = make_float4(G[c], G[c + 1], G[c + 2], G[c + 3]);
    }
}

// Sum of the slices' partials: dq, dk (input dtype), dg and dbeta (fp32).  One thread
// per (token, head, row); the slices are added in index order.
template <int D, typename TIn>
__global__ void __launch_bounds__(256)
kda_bwd_reduce_kernel(const float *__restrict__ part, long long ntok, int H,
                      TIn *__restrict__ dq, TIn *__restrict__ dk, float *__restrict__ dg,
                      float *__restrict__ dbeta) {
    constexpr int NS = D / SLC;
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long units = ntok * H;
    if (e >= units * (D + 1)) return;
    const long long u = e / (D + 1);
    const int r = (int)(e % (D + 1));
    const size_t pstride = (size_t)units * (3 * D + 1);
    if (r == D) {
        float s = 0.f;
        for (int sl = 0; sl < NS; ++sl) s += part[sl * pstride + (size_t)u * (3 * D + 1) + 3 * D];
        dbeta[u] = s;
        return;
    }
    float a = 0.f, b = 0.f, c = 0.f;
    for (int sl = 0; sl < NS; ++sl) {
        const float *pp = part + sl * pstride + (size_t)u * (3 * D + 1);
        a += pp[r];
        b += pp[D + r];
        c += pp[2 * D + r];
    }
    stf<TIn>(dq + (size_t)u * D + r, a);
    stf<TIn>(dk + (size_t)u * D + r, b);
    dg[(size_t)u * D + r] = c;
}

}  // namespace bwd
}  // namespace kda
