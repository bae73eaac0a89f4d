// kda_bwd_chain.cuh -- the chunk-level chain of the state gradient (backward pass).
//
// The forward's chunk records ("Kimi K3" open-weights field notes, panel "KDA 单头递归",
// taken 64 tokens at a time) give each chunk's affine map on the state,
//     S_out = P S_in + R,   O = Q' S_in + O0,   P = Diag(exp G_C) + M'.
// By the chain rule the loss gradient with respect to the state before the chunk is
//     dS_in = P^T dS_out + Q'^T dO = Diag(exp G_C) dS_out + M'^T dS_out + Q'^T dO,
// the forward state update with M'^T in place of M' and Q'^T dO in place of R.  The
// kernel below writes that "reverse record" for every (chunk, head), each sequence's
// chunks in reverse order, in the forward record's format; the state pass run over
// them from dL/dS_T then walks every sequence from its last chunk to its first, and
// its checkpoints are dL/dS at chunk boundaries: the ending gradients from which the
// per-token backward can run on every segment of a chain at once.
#pragma once

#include "kda_prefill_tc.cuh"

namespace kda {
namespace bwd {

constexpr int kRevThreads = 256;
constexpr int kRevPad = 8;   // bf16 elements of padding per shared-memory row

struct RevSmem {
    // bf16 bit patterns, row-major with padded rows (16-byte vector accesses by
    // consecutive rows do not share banks)
    uint16_t m[tc::D][tc::D + kRevPad];    // M'
    uint16_t qp[tc::C][tc::D + kRevPad];   // Q'
    uint16_t d[tc::C][tc::D + kRevPad];    // dO of the chunk's tokens (zero past the sequence)
};

// Reverse records of a fixed-length batch: item = chunk * H + head over B * cps chunks
// (cps = ceil(T / C) per sequence).  Record (n, j, h) goes to slot (n, cps - 1 - j, h).
// Every byte of the output record is written: M'^T, exp(G_C), R = Q'^T dO (fp32 sums of
// bf16 products, rounded to bf16), and zeros for Q' and O0.  Grid-stride over items.
__global__ void __launch_bounds__(kRevThreads)
kda_bwd_rev_records_kernel(const uint8_t *__restrict__ recs, const __nv_bfloat16 *__restrict__ dO,
                           uint8_t *__restrict__ rrec, int T, int H, int cps, long long items) {
    using namespace tc;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    RevSmem &sm = *reinterpret_cast<RevSmem *>(smem_raw);
    const int tid = threadIdx.x;
    for (long long item = blockIdx.x; item < items; item += gridDim.x) {
        const long long cid = item / H;
        const int h = (int)(item % H), n = (int)(cid / cps), j = (int)(cid % cps);
        const int len = min(C, T - j * C);
        const uint8_t *rec = recs + item * REC_BYTES;
        uint8_t *out = rrec + (((long long)n * cps + (cps - 1 - j)) * H + h) * REC_BYTES;
        // M' and Q' from the core-matrix layout (consecutive threads: consecutive rows,
        // contiguous in the record); the chunk's dO rows
        for (int x = tid; x < D * D / 8; x += kRevThreads) {
            const int r = x % D, c8 = x / D;
            *reinterpret_cast<uint4 *>(&sm.m[r][c8 * 8]) =
                *reinterpret_cast<const uint4 *>(rec + REC_M + core_off(D, r, c8 * 8));
        }
        for (int x = tid; x < C * D / 8; x += kRevThreads) {
            const int r = x % C, c8 = x / C;
            *reinterpret_cast<uint4 *>(&sm.qp[r][c8 * 8]) =
                *reinterpret_cast<const uint4 *>(rec + REC_QP + core_off(C, r, c8 * 8));
        }
        for (int x = tid; x < C * D / 8; x += kRevThreads) {
            const int r = x / (D / 8), c8 = x % (D / 8);
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (r < len)
                val = *reinterpret_cast<const uint4 *>(
                    dO + (((size_t)n * T + (size_t)j * C + r) * H + h) * D + c8 * 8);
            *reinterpret_cast<uint4 *>(&sm.d[r][c8 * 8]) = val;
        }
        __syncthreads();
        // M'^T: row i of the output holds column i of M'
        for (int x = tid; x < D * D / 8; x += kRevThreads) {
            const int i = x % D, c8 = x / D;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = (uint32_t)sm.m[c8 * 8 + 2 * e][i] | ((uint32_t)sm.m[c8 * 8 + 2 * e + 1][i] << 16);
            *reinterpret_cast<uint4 *>(out + REC_M + core_off(D, i, c8 * 8)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (tid < D * 4 / 16)
            reinterpret_cast<uint4 *>(out + REC_GC)[tid] =
                reinterpret_cast<const uint4 *>(rec + REC_GC)[tid];
        for (int x = tid; x < C * D * 2 / 16; x += kRevThreads) {
            reinterpret_cast<uint4 *>(out + REC_QP)[x] = make_uint4(0u, 0u, 0u, 0u);
            reinterpret_cast<uint4 *>(out + REC_O0)[x] = make_uint4(0u, 0u, 0u, 0u);
        }
        // R = Q'^T dO: thread -> key rows i0 .. i0 + 7, value columns c0 .. c0 + 7
        {
            const int i0 = (tid & 15) * 8, c0 = (tid >> 4) * 8;
            float acc[8][8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
            for (int r = 0; r < C; ++r) {
                const uint4 qa = *reinterpret_cast<const uint4 *>(&sm.qp[r][i0]);
                const uint4 da = *reinterpret_cast<const uint4 *>(&sm.d[r][c0]);
                const uint32_t qw[4] = {qa.x, qa.y, qa.z, qa.w}, dw[4] = {da.x, da.y, da.z, da.w};
                float qf[8], df[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = unpack_bf16x2(qw[e]), y = unpack_bf16x2(dw[e]);
                    qf[2 * e] = x.x;
                    qf[2 * e + 1] = x.y;
                    df[2 * e] = y.x;
                    df[2 * e + 1] = y.y;
                }
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(qf[a], df[b], acc[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                uint4 pk;
                pk.x = pack_bf16x2(acc[a][0], acc[a][1]);
                pk.y = pack_bf16x2(acc[a][2], acc[a][3]);
                pk.z = pack_bf16x2(acc[a][4], acc[a][5]);
                pk.w = pack_bf16x2(acc[a][6], acc[a][7]);
                *reinterpret_cast<uint4 *>(out + REC_R + core_off(D, i0 + a, c0)) = pk;
            }
        }
        __syncthreads();   // the next item overwrites the tiles
    }
}

}  // namespace bwd
}  // namespace kda
