// kda_decode.cuh -- one-token KDA decode step, state updated in place.
//
// For each (sequence, head), with the recurrence of the "Kimi K3" open-weights
// field notes (panel "KDA 单头递归") at T = 1:
//   S' = Diag(exp g) S;   p = S'^T k;   r = S'^T q;   delta = b (v - p)
//   S  = S' + k delta^T;  o = S^T q = r + (k . q) delta
// The state is read from HBM once and written once: it streams through
// registers as float4 column groups (a warp covers whole 512-byte rows when
// d_v = 128), and the two column reductions over key rows go through shared
// memory.  One CTA per (sequence, head); the kernel is bound by HBM bandwidth.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace dec {

constexpr int NT = 256;

template <typename TIn>
KDA_DEVINL float ld1(const TIn *p);
template <>
KDA_DEVINL float ld1<float>(const float *p) { return __ldg(p); }
template <>
KDA_DEVINL float ld1<__nv_bfloat16>(const __nv_bfloat16 *p) { return bf2f(*p); }

// RPT consecutive fp32 values of a shared-memory row (16-byte aligned when RPT is a
// multiple of 4), as few vector loads as possible.
template <int RPT>
KDA_DEVINL void ld_rows(const float *p, float (&x)[RPT]) {
    if constexpr (RPT % 4 == 0) {
#pragma unroll
        for (int i = 0; i < RPT; i += 4) {
            const float4 v = *reinterpret_cast<const float4 *>(p + i);
            x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < RPT; ++i) x[i] = p[i];
    }
}

template <int D, typename TIn>
__global__ void __launch_bounds__(NT, 2)
kda_decode_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                  const TIn *__restrict__ v, const float *__restrict__ g,
                  const float *__restrict__ beta, float *__restrict__ S,
                  TIn *__restrict__ o) {
    constexpr int CG = D / 4;        // float4 column groups per row
    constexpr int RS = NT / CG;      // row slots
    constexpr int RPT = D / RS;      // rows per thread
    static_assert(NT % CG == 0 && D % RS == 0, "thread mapping");
    __shared__ float s_k[D], s_q[D], s_a[D];
    __shared__ __align__(16) float s_p[RS][D];
    __shared__ __align__(16) float s_r[RS][D];
    __shared__ __align__(16) float s_delta[D];
    __shared__ float s_kq;

    const int tid = threadIdx.x;
    const int cg = tid % CG, rs = tid / CG;
    const size_t unit = blockIdx.x;                 // (sequence, head)
    float4 *Sp = reinterpret_cast<float4 *>(S + unit * D * D);

    // Issue every state load first: RPT independent 16-byte loads per thread.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(Sp + (rs * RPT + i) * CG + cg);

    if (tid < D) {
        s_k[tid] = ld1<TIn>(k + unit * D + tid);
        s_q[tid] = ld1<TIn>(q + unit * D + tid);
        s_a[tid] = expf(__ldg(g + unit * D + tid));
    }
    __syncthreads();
    if (tid < 32) {
        float x = 0.f;
        for (int i = tid; i < D; i += 32) x += s_k[i] * s_q[i];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
        if (tid == 0) s_kq = x;
    }
    // decay, then partial column sums of k^T S' and q^T S' over this thread's rows
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
    float av[RPT], kv[RPT], qv[RPT];   // this thread's rows rs RPT .. rs RPT + RPT - 1
    ld_rows<RPT>(&s_a[rs * RPT], av);
    ld_rows<RPT>(&s_k[rs * RPT], kv);
    ld_rows<RPT>(&s_q[rs * RPT], qv);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float a = av[i], kr = kv[i], qr = qv[i];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk.x += kr * s[i].x; pk.y += kr * s[i].y; pk.z += kr * s[i].z; pk.w += kr * s[i].w;
        pq.x += qr * s[i].x; pq.y += qr * s[i].y; pq.z += qr * s[i].z; pq.w += qr * s[i].w;
    }
    *reinterpret_cast<float4 *>(&s_p[rs][cg * 4]) = pk;
    *reinterpret_cast<float4 *>(&s_r[rs][cg * 4]) = pq;
    __syncthreads();
    if (tid < D) {
        float p = 0.f, r = 0.f;
#pragma unroll
        for (int j = 0; j < RS; ++j) {
            p += s_p[j][tid];
            r += s_r[j][tid];
        }
        const float b = __ldg(beta + unit);
        const float d = b * (ld1<TIn>(v + unit * D + tid) - p);
        s_delta[tid] = d;
        const float out = r + s_kq * d;
        if constexpr (sizeof(TIn) == 2)
            o[unit * D + tid] = f2bf(out);
        else
            o[unit * D + tid] = out;
    }
    __syncthreads();
    const float4 dl = *reinterpret_cast<const float4 *>(&s_delta[cg * 4]);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kr = kv[i];
        s[i].x += kr * dl.x; s[i].y += kr * dl.y; s[i].z += kr * dl.z; s[i].w += kr * dl.w;
        __stcs(Sp + (rs * RPT + i) * CG + cg, s[i]);
    }
}

// ---------------------------------------------------------------------------
// Speculative decoding: verify K drafted tokens, then commit the accepted prefix.
//
// A draft proposes K tokens per sequence; the target model runs them as one small
// batch and accepts a prefix of a <= K of them ("Kimi K3" open-weights field notes,
// panel "目标模型太大，缓存和草稿都必须理解 KDA": the draft and the cache must follow
// the KDA state, a rejected draft must not leave its tokens in the state, and the
// accepted states are replayed on chip from the cached projected inputs).
//   verify: from S, run the K tokens of the recurrence in registers and write the
//           K outputs; S is only read (one HBM read of the state).
//   commit: from S, replay the first a_n tokens (a_n from the device array
//           `accepted`) and write the state back (one read and one write); a_n = 0
//           leaves S untouched, a_n outside [0, K] sets the error bit and leaves S
//           untouched.
// Layouts: q, k, g [N, K, H, D]; v, o [N, K, H, D]; beta [N, K, H]; S [N, H, D, D].
// Same thread mapping as kda_decode_kernel (float4 column groups, RPT rows per
// thread); a token's inputs are staged in shared memory up front.
// ---------------------------------------------------------------------------
constexpr int kMaxDraft = 16;        // largest K
constexpr int kErrAcceptedBit = 16;  // device error word: an accepted count out of range

template <int D, typename TIn, bool COMMIT>
__global__ void __launch_bounds__(NT, 2)
kda_decode_multi_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                        const TIn *__restrict__ v, const float *__restrict__ g,
                        const float *__restrict__ beta, float *__restrict__ S,
                        TIn *__restrict__ o, const int *__restrict__ accepted, int K, int H,
                        int *err_word) {
    constexpr int CG = D / 4, RS = NT / CG, RPT = D / RS;
    static_assert(NT % CG == 0 && D % RS == 0, "thread mapping");
    __shared__ float s_k[kMaxDraft][D], s_a[kMaxDraft][D], s_v[kMaxDraft][D];
    __shared__ float s_q[COMMIT ? 1 : kMaxDraft][D];
    __shared__ float s_b[kMaxDraft], s_kq[kMaxDraft];
    __shared__ __align__(16) float s_p[RS][D];
    __shared__ __align__(16) float s_r[COMMIT ? 1 : RS][D];
    __shared__ __align__(16) float s_delta[D];

    const int tid = threadIdx.x, cg = tid % CG, rs = tid / CG;
    const size_t unit = blockIdx.x;                 // (sequence, head)
    const int n = (int)(unit / H), h = (int)(unit % H);
    int ntok = K;
    if constexpr (COMMIT) {
        ntok = accepted[n];
        if (ntok < 0 || ntok > K) {
            if (tid == 0 && h == 0) atomicOr(err_word, kErrAcceptedBit);
            return;
        }
        if (ntok == 0) return;   // nothing accepted: the state stays as it is
    }
    float4 *Sp = reinterpret_cast<float4 *>(S + unit * D * D);
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(Sp + (rs * RPT + i) * CG + cg);

    // stage the tokens' inputs: token t of (n, h) sits at row (n K + t) H + h
    for (int e = tid; e < ntok * D; e += NT) {
        const int t = e / D, c = e % D;
        const size_t row = ((size_t)n * K + t) * H + h;
        s_k[t][c] = ld1<TIn>(k + row * D + c);
        s_a[t][c] = expf(__ldg(g + row * D + c));
        s_v[t][c] = ld1<TIn>(v + row * D + c);
        if constexpr (!COMMIT) s_q[t][c] = ld1<TIn>(q + row * D + c);
    }
    if (tid < ntok) s_b[tid] = __ldg(beta + ((size_t)n * K + tid) * H + h);
    __syncthreads();
    if constexpr (!COMMIT) {   // k_t . q_t, one warp per token
        for (int t = tid >> 5; t < ntok; t += NT / 32) {
            float x = 0.f;
            for (int i = tid & 31; i < D; i += 32) x += s_k[t][i] * s_q[t][i];
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
            if ((tid & 31) == 0) s_kq[t] = x;
        }
    }
    for (int t = 0; t < ntok; ++t) {
        // decay, then partial column sums of k^T S' (and q^T S') over this thread's rows
        float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
        float av[RPT], kv[RPT], qv[COMMIT ? 1 : RPT];   // rows rs RPT .. rs RPT + RPT - 1
        ld_rows<RPT>(&s_a[t][rs * RPT], av);
        ld_rows<RPT>(&s_k[t][rs * RPT], kv);
        if constexpr (!COMMIT) ld_rows<RPT>(&s_q[t][rs * RPT], qv);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float a = av[i], kr = kv[i];
            s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
            pk.x += kr * s[i].x; pk.y += kr * s[i].y; pk.z += kr * s[i].z; pk.w += kr * s[i].w;
            if constexpr (!COMMIT) {
                const float qr = qv[i];
                pq.x += qr * s[i].x; pq.y += qr * s[i].y; pq.z += qr * s[i].z; pq.w += qr * s[i].w;
            }
        }
        *reinterpret_cast<float4 *>(&s_p[rs][cg * 4]) = pk;
        if constexpr (!COMMIT) *reinterpret_cast<float4 *>(&s_r[rs][cg * 4]) = pq;
        __syncthreads();
        if (tid < D) {
            float p = 0.f, r = 0.f;
#pragma unroll
            for (int j = 0; j < RS; ++j) {
                p += s_p[j][tid];
                if constexpr (!COMMIT) r += s_r[j][tid];
            }
            const float d = s_b[t] * (s_v[t][tid] - p);
            s_delta[tid] = d;
            if constexpr (!COMMIT) {
                const float out = r + s_kq[t] * d;
                const size_t row = ((size_t)n * K + t) * H + h;
                if constexpr (sizeof(TIn) == 2)
                    o[row * D + tid] = f2bf(out);
                else
                    o[row * D + tid] = out;
            }
        }
        __syncthreads();
        const float4 dl = *reinterpret_cast<const float4 *>(&s_delta[cg * 4]);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float kr = kv[i];
            s[i].x += kr * dl.x; s[i].y += kr * dl.y; s[i].z += kr * dl.z; s[i].w += kr * dl.w;
        }
    }
    if constexpr (COMMIT) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) __stcs(Sp + (rs * RPT + i) * CG + cg, s[i]);
    }
}

}  // namespace dec
}  // namespace kda
