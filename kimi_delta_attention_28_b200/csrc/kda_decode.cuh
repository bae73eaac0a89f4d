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
    for (int i = 0; i < RPT; ++i) s[i] = __ldcs(Sp + (rs + i * RS) * CG + cg);

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
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int row = rs + i * RS;
        const float a = s_a[row], kr = s_k[row], qr = s_q[row];
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
        const int row = rs + i * RS;
        const float kr = s_k[row];
        s[i].x += kr * dl.x; s[i].y += kr * dl.y; s[i].z += kr * dl.z; s[i].w += kr * dl.w;
        __stcs(Sp + row * CG + cg, s[i]);
    }
}

}  // namespace dec
}  // namespace kda
