// kda_common.cuh -- device helpers shared by the KDA kernels (sm_100a).
//
// Warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulate), ldmatrix
// fragment loads, cp.async copies and bf16 packing.  Fragment layouts follow
// the PTX ISA description of mma.m16n8k16 (A row-major, B column-major):
//   lane = 4*gid + tig;  A regs: (gid, 2tig..), (gid+8, 2tig..), (gid, 2tig+8..),
//   (gid+8, 2tig+8..);  B regs: (k=2tig.., n=gid), (k=2tig+8.., n=gid);
//   C regs: (gid, 2tig), (gid, 2tig+1), (gid+8, 2tig), (gid+8, 2tig+1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KDA_DEVINL __device__ __forceinline__

namespace kda {

constexpr float kLog2e = 1.4426950408889634f;

KDA_DEVINL uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

KDA_DEVINL float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }
KDA_DEVINL __nv_bfloat16 f2bf(float x) { return __float2bfloat16_rn(x); }

// Pack two floats into a bf16x2 register (lo in the low half), RNE.
KDA_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
KDA_DEVINL float2 unpack_bf16x2(uint32_t v) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162 *>(&v);
    return __bfloat1622float2(b);
}

// D += A * B, bf16 inputs, fp32 accumulators.
KDA_DEVINL void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

KDA_DEVINL void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
KDA_DEVINL void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// 16-byte async global->shared copy; src_bytes < 16 zero-fills the remainder.
KDA_DEVINL void cp_async16(void *smem, const void *gmem, int src_bytes = 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(src_bytes));
}
KDA_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
KDA_DEVINL void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ---- fragment address helpers (element offsets inside a row-major smem tile) ----
// A fragment (16x16) of a row-major [M][K] tile at (m0, k0).
KDA_DEVINL int frag_a_row(int lane) { return lane & 15; }
KDA_DEVINL int frag_a_col(int lane) { return (lane >> 4) << 3; }
// A fragment from a tile stored transposed, [K][M] row-major (ldmatrix.trans).
KDA_DEVINL int frag_at_row(int lane) { return (lane & 7) + ((lane >> 4) << 3); }  // k offset
KDA_DEVINL int frag_at_col(int lane) { return ((lane >> 3) & 1) << 3; }            // m offset
// Two B fragments (n-tiles n0, n0+8) from a tile stored [N][K] row-major (ldmatrix).
KDA_DEVINL int frag_bn_row(int lane) { return (lane & 7) + ((lane >> 4) << 3); }   // n offset
KDA_DEVINL int frag_bn_col(int lane) { return ((lane >> 3) & 1) << 3; }            // k offset
// Two B fragments (n-tiles n0, n0+8) from a tile stored [K][N] row-major (ldmatrix.trans).
KDA_DEVINL int frag_bk_row(int lane) { return (lane & 7) + (((lane >> 3) & 1) << 3); }  // k off
KDA_DEVINL int frag_bk_col(int lane) { return (lane >> 4) << 3; }                       // n off

}  // namespace kda

namespace kda {

// ---- mbarrier / bulk-copy (TMA engine) primitives ----
KDA_DEVINL void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
KDA_DEVINL void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::); }
KDA_DEVINL void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::); }
KDA_DEVINL void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
KDA_DEVINL bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
KDA_DEVINL uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
    return t;
}
// Wait for the barrier phase with a wall-clock limit.  Returns false on timeout.
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
KDA_DEVINL bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
KDA_DEVINL void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
        ::"r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---- swizzled tile layouts (16-byte chunks XOR-permuted by row) ----
// Byte offset of bf16 element (r, c) in a [rows][128] tile with 256-byte rows.
KDA_DEVINL int swz128(int r, int c) { return r * 256 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1); }
// Byte offset of bf16 element (r, c) in a [rows][64] tile with 128-byte rows.
KDA_DEVINL int swz64(int r, int c) { return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1); }

}  // namespace kda

namespace kda {
// Byte offset of bf16 element (r, c) in a [rows][256] tile with 512-byte rows.
KDA_DEVINL int swz256(int r, int c) { return r * 512 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1); }
}  // namespace kda
