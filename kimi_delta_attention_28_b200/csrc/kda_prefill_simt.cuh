// kda_prefill_simt.cuh -- chunkwise KDA prefill in fp32 on CUDA cores.
//
// Serves fp32 inputs (where bf16 tensor-core operands would miss a 1e-4
// relative tolerance) and the small head sizes 32 and 64.  Same chunk algebra as
// the tensor-core path (see kda_prefill_tc.cuh), with a 16-token chunk, every
// product in fp32, and the pairwise decays exp(G_r - G_i) (i <= r, so <= 1)
// evaluated directly.  One CTA per (sequence, head) walks its chunks in order
// with the d_k x d_v state in shared memory.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace simt {

constexpr int C = 16;
constexpr int NT = 256;   // threads per CTA

template <typename TIn>
KDA_DEVINL float ld_in(const TIn *p);
template <>
KDA_DEVINL float ld_in<float>(const float *p) { return *p; }
template <>
KDA_DEVINL float ld_in<__nv_bfloat16>(const __nv_bfloat16 *p) { return bf2f(*p); }
template <typename TIn>
KDA_DEVINL void st_out(TIn *p, float x);
template <>
KDA_DEVINL void st_out<float>(float *p, float x) { *p = x; }
template <>
KDA_DEVINL void st_out<__nv_bfloat16>(__nv_bfloat16 *p, float x) { *p = f2bf(x); }

template <int D>
struct SimtSmem {
    float S[D * D];      // state, row = key channel, column = value channel
    float q[C * D];      // queries, then q * exp(G)
    float k[C * D];      // keys, then k * exp(G_C - G)
    float v[C * D];
    float G[C * D];      // inclusive cumulative log-decay (natural units)
    float w[C * D];      // W
    float u[C * D];      // U, then Delta
    float akk[C * (C + 1)];
    float aqk[C * (C + 1)];
    float beta[C];
    float gC[D];         // exp(G_C)
};

template <int D, typename TIn>
__global__ void __launch_bounds__(NT)
kda_simt_fwd_kernel(const TIn *__restrict__ q, const TIn *__restrict__ k,
                    const TIn *__restrict__ v, const float *__restrict__ g,
                    const float *__restrict__ beta, const float *h0, float *hT,
                    TIn *__restrict__ o, int T, int H, const int *__restrict__ hdr,
                    const int *__restrict__ cu, long long ntok, int *err_word) {
    static_assert(NT % D == 0, "thread mapping");
    constexpr int RG = NT / D;   // row groups
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SimtSmem<D> &sm = *reinterpret_cast<SimtSmem<D> *>(smem_raw);
    const int tid = threadIdx.x;
    const int chain = blockIdx.x, n = chain / H, h = chain % H;
    int seq_t0, seq_len;
    if (cu) {
        if (!hdr[0]) return;
        seq_t0 = cu[n];
        seq_len = cu[n + 1] - cu[n];
    } else {
        seq_t0 = n * T;
        seq_len = T;
    }
    if constexpr (KDA_DEBUG) {   // the sequence's tokens inside q, k, v, g, beta and o
        if (seq_len < 0 || seq_t0 < 0 || (long long)seq_t0 + seq_len > ntok) {
            if (tid == 0) atomicOr(err_word, kErrBoundsBit);
            return;
        }
    }
    const size_t sbase = (size_t)chain * D * D;
    for (int e = tid; e < D * D; e += NT) sm.S[e] = h0 ? h0[sbase + e] : 0.f;
    __syncthreads();

    const int jcol = tid % D, rg = tid / D;
    for (int c0 = 0; c0 < seq_len; c0 += C) {
        const int len = min(C, seq_len - c0);
        const size_t base = ((size_t)(seq_t0 + c0) * H + h) * D;
        const size_t rs = (size_t)H * D;
        for (int e = tid; e < C * D; e += NT) {
            const int r = e / D, c = e % D;
            const bool ok = r < len;
            sm.q[e] = ok ? ld_in<TIn>(q + base + r * rs + c) : 0.f;
            sm.k[e] = ok ? ld_in<TIn>(k + base + r * rs + c) : 0.f;
            sm.v[e] = ok ? ld_in<TIn>(v + base + r * rs + c) : 0.f;
            sm.G[e] = ok ? g[base + r * rs + c] : 0.f;
        }
        if (tid < C) sm.beta[tid] = tid < len ? beta[(size_t)(seq_t0 + c0 + tid) * H + h] : 0.f;
        __syncthreads();
        if (tid < D) {   // inclusive cumsum over the chunk, one channel per thread
            float run = 0.f;
            for (int r = 0; r < C; ++r) {
                run += sm.G[r * D + tid];
                sm.G[r * D + tid] = run;
            }
            sm.gC[tid] = expf(run);
        }
        __syncthreads();
        // A_kk (strictly lower, times beta_r) and A_qk (lower incl. diagonal)
        for (int p = tid; p < C * C; p += NT) {
            const int r = p / C, i = p % C;
            float akk = 0.f, aqk = 0.f;
            if (i <= r) {
                for (int c = 0; c < D; ++c) {
                    const float e = expf(sm.G[r * D + c] - sm.G[i * D + c]);
                    const float ki = sm.k[i * D + c] * e;
                    akk += sm.k[r * D + c] * ki;
                    aqk += sm.q[r * D + c] * ki;
                }
            }
            sm.akk[r * (C + 1) + i] = (i < r) ? akk * sm.beta[r] : 0.f;
            sm.aqk[r * (C + 1) + i] = aqk;
        }
        __syncthreads();
        // W = (I+A)^-1 Diag(b)(K*exp G), U = (I+A)^-1 Diag(b) V: forward substitution,
        // one column per thread.
        for (int col = tid; col < 2 * D; col += NT) {
            const int c = col % D;
            const bool isW = col < D;
            float *dst = isW ? sm.w : sm.u;
            for (int r = 0; r < C; ++r) {
                float x = sm.beta[r] * (isW ? sm.k[r * D + c] * expf(sm.G[r * D + c])
                                            : sm.v[r * D + c]);
                for (int i = 0; i < r; ++i) x -= sm.akk[r * (C + 1) + i] * dst[i * D + c];
                dst[r * D + c] = x;
            }
        }
        __syncthreads();
        // Delta = U - W S (in place over U)
        for (int r = rg; r < C; r += RG) {
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc += sm.w[r * D + c] * sm.S[c * D + jcol];
            sm.u[r * D + jcol] -= acc;
        }
        // queries -> q * exp(G), keys -> k * exp(G_C - G)
        for (int e = tid; e < C * D; e += NT) {
            const int c = e % D;
            const float Gr = sm.G[e];
            const float GC = sm.G[(C - 1) * D + c];
            sm.q[e] *= expf(Gr);
            sm.k[e] *= expf(GC - Gr);
        }
        __syncthreads();
        // O = (Q*exp G) S + A_qk Delta
        for (int r = rg; r < C; r += RG) {
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc += sm.q[r * D + c] * sm.S[c * D + jcol];
            for (int i = 0; i <= r; ++i) acc += sm.aqk[r * (C + 1) + i] * sm.u[i * D + jcol];
            if (r < len) st_out<TIn>(o + base + r * rs + jcol, acc);
        }
        __syncthreads();
        // S = Diag(exp G_C) S + (K*exp(G_C - G))^T Delta
        for (int c = rg; c < D; c += RG) {
            float acc = sm.gC[c] * sm.S[c * D + jcol];
            for (int r = 0; r < C; ++r) acc += sm.k[r * D + c] * sm.u[r * D + jcol];
            sm.S[c * D + jcol] = acc;
        }
        __syncthreads();
    }
    if (hT)
        for (int e = tid; e < D * D; e += NT) hT[sbase + e] = sm.S[e];
}

}  // namespace simt
}  // namespace kda
