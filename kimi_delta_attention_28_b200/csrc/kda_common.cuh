// kda_common.cuh -- device helpers shared by the KDA kernels (sm_100a).
//
// Warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulate), ldmatrix
// fragment loads, cp.async copies and bf16 packing.  Fragment layouts follow
// the PTX ISA description of mma.m16n8k16 (A row-major, B column-major):
//   lane = 4*gid + tig;  A regs: (gid, 2tig..), (gid+8, 2tig..), (gid, 2tig+8..),
//   (gid+8, 2tig+8..);  B regs: (k=2tig.., n=gid), (k=2tig+8.., n=gid);
//   C regs: (gid, 2tig), (gid, 2tig+1), (gid+8, 2tig), (gid+8, 2tig+1).
#pragma once

#include <cuda.h>   // CUtensorMap (the type only; maps are encoded through the runtime's
                    // driver entry points)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define KDA_DEVINL __device__ __forceinline__

// Debug builds (-DKDA_DEBUG=1, the library libkda_b200_debug.so) check, at the top
// of every prefill kernel, the indices that address global memory -- chunk table
// entries, sequence ranges, record slots -- against the extents of their buffers.
// A failed check sets the bounds bit of the device error word and the CTA returns
// before its first access, instead of faulting.  Release builds compile them out.
#ifndef KDA_DEBUG
#define KDA_DEBUG 0
#endif

namespace kda {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kErrBoundsBit = 8;   // device error word: a debug bounds check failed

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


// Four 8x8 bf16 tiles from registers to shared memory, each stored transposed:
// lanes 8m..8m+7 give the row addresses of tile m (register m), and thread t's pair
// (row t/4, columns 2(t%4), 2(t%4)+1) of the tile lands in rows 2(t%4), 2(t%4)+1,
// column t/4.
KDA_DEVINL void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};\n"
                 ::"r"(addr), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

// 2^x by the PTX instruction ex2.approx.ftz.f32 (relative error about 2^-22;
// results below the normal fp32 range flush to zero).
KDA_DEVINL float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// 16-byte async global->shared copy; src_bytes < 16 zero-fills the remainder.
KDA_DEVINL void cp_async16(void *smem, const void *gmem, int src_bytes = 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(src_bytes));
}
// 4-byte async global->shared copy (cp.async.ca); src_bytes = 0 writes zero.
KDA_DEVINL void cp_async4(void *smem, const void *gmem, int src_bytes = 4) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(smem)),
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
// Plain arrival (release, CTA scope) on a count-initialised barrier.
KDA_DEVINL void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
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

// ---- named CTA barriers (a group of `n` threads, a multiple of 32, on barrier `id`) ----
// With id 0 and n = the block size these are __syncthreads and its reductions; other
// ids let independent thread groups of one CTA synchronise among themselves.
KDA_DEVINL void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
KDA_DEVINL bool bar_and(int id, int n, bool p) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
                 " bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
                 : "=r"(r) : "r"((uint32_t)p), "r"(id), "r"(n) : "memory");
    return r != 0;
}
KDA_DEVINL bool bar_or(int id, int n, bool p) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
                 " bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
                 : "=r"(r) : "r"((uint32_t)p), "r"(id), "r"(n) : "memory");
    return r != 0;
}

// ---- flags between CTAs of one launch (GPU scope) ----
// Generic-proxy accesses of global memory before this fence are ordered with this
// thread's later asynchronous-proxy (bulk copy) accesses, and the other way round.
KDA_DEVINL void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;\n" ::: "memory"); }
KDA_DEVINL void flag_release(int *f, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(f), "r"(v) : "memory");
}
// A counter another CTA only reads as a hint (no ordering with other accesses).
KDA_DEVINL void store_relaxed(int *f, int v) {
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;\n" ::"l"(f), "r"(v) : "memory");
}
KDA_DEVINL int flag_acquire(const int *f) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(f) : "memory");
    return v;
}
// Wait until *f != 0, with the same wall-clock limit as the barrier waits.
KDA_DEVINL bool flag_wait_bounded(const int *f) {
    if (flag_acquire(f)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!flag_acquire(f)) {
        __nanosleep(64);
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}
// Tiled 4-D tensor copy global -> this CTA's shared memory by the tensor-memory-access
// engine, completing on `bar`: the box of the tensor map `tm` at coordinates
// (c0, c1, c2, c3), innermost first.  Coordinates past the tensor's extent read zeros.
// No cluster multicast.
KDA_DEVINL void tma_load_4d(void *smem_dst, const CUtensorMap *tm, int c0, int c1, int c2,
                            int c3, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];\n"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1),
          "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
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

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core) helpers, sm_100a.
// ---------------------------------------------------------------------------
namespace kda {
namespace t5 {

// Shared-memory matrix descriptor: start address (>>4) in bits [0,14), leading
// byte offset (>>4) in [16,30), stride byte offset (>>4) in [32,46), descriptor
// version 1 in [46,48), swizzle mode in [61,64) (2 = 128-byte, 4 = 64-byte).
KDA_DEVINL uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                              uint32_t swizzle) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)(swizzle & 7) << 61;
    return d;
}
constexpr uint32_t kSwz128 = 2, kSwz64 = 4;

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
// a_mn / b_mn: 1 when that operand is MN-major (M or N contiguous), 0 when K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                          // D format: f32
           | (1u << 7) | (1u << 10)           // A, B format: bf16
           | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16)
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

KDA_DEVINL void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread is done.
KDA_DEVINL void commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
                 ::"r"(smem_u32(bar))
                 : "memory");
}
// One lane of the (fully active) warp returns true.
KDA_DEVINL bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n .reg .pred p;\n elect.sync _|p, 0xffffffff;\n selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(pred));
    return pred != 0;
}
KDA_DEVINL void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
KDA_DEVINL void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
// Whole-warp TMEM allocation; the base address is written to *dst (shared memory).
KDA_DEVINL void alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
KDA_DEVINL void relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
KDA_DEVINL void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (32x32b shape, x32).  The
// wait is in the same statement, so the outputs are defined when it returns.
KDA_DEVINL void ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive fp32 columns of this thread's TMEM lane (32x32b shape, x64), wait included.
KDA_DEVINL void ld64(uint32_t taddr, float (&v)[64]) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}
// 16x256b shape, x4: lanes L..L+15 of this warp's quarter (L from taddr) and 32
// columns.  Thread t (g = t/4, c = t%4) receives, for each 8-column group j (0..3),
// v[4j], v[4j+1] = (lane L+g, columns 8j+2c, 8j+2c+1) and v[4j+2], v[4j+3] = the same
// columns of lane L+g+8 -- the mma.sync accumulator layout; for an M = 64 accumulator
// (rows 16w..16w+15 in lanes 32w..32w+15) every thread of the warp gets data.
KDA_DEVINL void ld16x256b_x4(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
template <int N>
KDA_DEVINL void ld_cols(uint32_t taddr, float (&v)[N]) {
    if constexpr (N == 32) ld32(taddr, v);
    else ld64(taddr, v);
}

}  // namespace t5
}  // namespace kda
