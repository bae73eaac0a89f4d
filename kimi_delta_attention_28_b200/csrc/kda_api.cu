// kda_api.cu -- the library's C ABI (declared in include/kda.h).
//
// Host-side argument validation, workspace layout and kernel dispatch.  All
// kernels are compiled into this one translation unit so they can share the
// device error word without relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/kda.h"
#include "kda_bwd.cuh"
#include "kda_bwd_chain.cuh"
#include "kda_common.cuh"
#include "kda_decode.cuh"
#include "kda_prefill_simt.cuh"
#include "kda_prefill_tc.cuh"

// Sticky device error bits; read and cleared by kda_get_last_device_error.
__device__ int g_kda_device_error = 0;

namespace {

constexpr int ERRBIT_SEQLENS = 1;
constexpr int ERRBIT_TIMEOUT = 2;
constexpr int ERRBIT_CKPT = 4;
constexpr int ERRBIT_BOUNDS = kda::kErrBoundsBit;
constexpr int ERRBIT_ACCEPTED = kda::dec::kErrAcceptedBit;

inline bool aligned_to(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;  // NULL counts as aligned
}
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout of kda_fwd (all segments 256-byte aligned):
//   header   : 2 ints (offsets-valid flag, total chunks)
//   seq_off  : num_seqs + 1 ints
//   chunks   : max_chunks ChunkLoc
//   records  : max_chunks * H records of tc::REC_BYTES (tensor-core path only)
//   s_in     : (T-split only) units * D * D fp32 segment starting states
//   seg_map  : (T-split only) units * D * 2D fp32 segment maps [R | P]
// where units = chains (N * H) * nseg.
struct WsLayout {
    size_t hdr, seq_off, chunks, recs, ready, prog, s_in, seg_map, total;
    long long max_chunks;
    int nseg;
};

inline bool is_tc_path(int dtype, int dk) { return dtype == KDA_DTYPE_BF16 && dk == 128; }

// T-split policy.  Splitting a chain into nseg segments costs about three times
// its state-pass work (the map pass carries 2D columns, the output pass D) but
// runs nseg times as many CTAs, so it pays only when the unsplit pass leaves most
// SMs idle.  nseg is chosen so the map pass (chains * nseg * 2D/32 CTAs) fills at
// most one wave, with at least kMinSegChunks chunks per segment.
constexpr int kMaxSegments = 32;
constexpr int kMinSegChunks = 16;
constexpr int kSplitSmBound = 192;   // workspace sizing assumes at most this many SMs
constexpr int kProgressSlots = kSplitSmBound;   // state CTAs of the overlapped schedule
constexpr int kMaxSegmentsExplicit = 4096;   // cap of kda_fwd_segmented's num_segments

int split_segments(long long chains, long long chunks_per_chain, int sms) {
    if (chains <= 0 || sms <= 0) return 1;
    long long n = (long long)sms / (chains * (2 * kda::tc::D / 32));
    n = n < chunks_per_chain / kMinSegChunks ? n : chunks_per_chain / kMinSegChunks;
    n = n < kMaxSegments ? n : kMaxSegments;
    return n >= 2 ? (int)n : 1;
}

long long chunks_per_chain(int B, int T, int num_seqs, long long max_chunks) {
    if (num_seqs > 0) return max_chunks / num_seqs;   // packed: the mean
    (void)B;
    return ((long long)T + kda::tc::C - 1) / kda::tc::C;
}

// SM count of the current device, capped at kSplitSmBound (0 if unknown).
int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n < kSplitSmBound ? n : kSplitSmBound;
}

// nseg > 0: that many segments (tensor-core path); nseg == 0: the policy with
// `sms` multiprocessors.
WsLayout ws_layout(int B, int T, int H, int dk, int num_seqs, int dtype, int nseg = 0,
                   int sms = kSplitSmBound) {
    WsLayout L{};
    const bool varlen = num_seqs > 0;
    const int chunk = is_tc_path(dtype, dk) ? kda::tc::C : kda::simt::C;
    if (varlen)
        L.max_chunks = ((long long)T + chunk - 1) / chunk + num_seqs;
    else
        L.max_chunks = (long long)B * (((long long)T + chunk - 1) / chunk);
    L.hdr = 0;
    L.seq_off = 256;
    L.chunks = round_up(L.seq_off + sizeof(int) * (size_t)(num_seqs + 1), 256);
    L.recs = round_up(L.chunks + (varlen ? sizeof(kda::tc::ChunkLoc) * (size_t)L.max_chunks : 0),
                      256);
    L.total = L.recs;
    L.nseg = 1;
    if (is_tc_path(dtype, dk)) {
        L.total += (size_t)L.max_chunks * H * kda::tc::REC_BYTES;
        // the overlapped schedule's per-record ready flags and per-CTA progress counters
        L.ready = round_up(L.total, 256);
        L.prog = L.ready + (size_t)L.max_chunks * H * sizeof(int);
        L.total = L.prog + kProgressSlots * kda::tc::kProgStride * sizeof(int);
        const long long N = num_seqs > 0 ? num_seqs : B;
        L.nseg = nseg > 0 ? nseg
                          : split_segments(N * H, chunks_per_chain(B, T, num_seqs, L.max_chunks), sms);
        if (L.nseg > 1) {
            const size_t units = (size_t)N * H * L.nseg, D = kda::tc::D;
            L.s_in = round_up(L.total, 256);
            L.seg_map = round_up(L.s_in + units * D * D * sizeof(float), 256);
            L.total = L.seg_map + units * D * 2 * D * sizeof(float);
        }
    }
    return L;
}

kda_status check_shape(int H, int dk, int dv, int dtype) {
    if (H <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (dk != dv) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (dk != 32 && dk != 64 && dk != 128) return KDA_ERR_UNSUPPORTED_SHAPE;
    return KDA_OK;
}

int *device_error_word() {
    int *p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_kda_device_error) != cudaSuccess)
        return nullptr;
    return p;
}

// Test hook: KDA_TEST_DROP_FIRST_COPY=1 (read once per process) makes the state
// pass skip the bulk copy of its first chunk, so its bounded wait runs out and
// the call reports KDA_ERR_DEVICE_TIMEOUT.  Used only by the failure-path test.
int debug_drop_first_copy() {
    static const int v = [] {
        const char *e = getenv("KDA_TEST_DROP_FIRST_COPY");
        return (e && atoi(e) != 0) ? 1 : 0;
    }();
    return v;
}

kda_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <int D, typename TIn>
kda_status launch_simt(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *h0, float *hT, void *o, int T, int H,
                       int nunits, const int *hdr, const int *cu, long long ntok,
                       cudaStream_t s) {
    const size_t smem = sizeof(kda::simt::SimtSmem<D>);
    auto kern = kda::simt::kda_simt_fwd_kernel<D, TIn>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KDA_ERR_CUDA;
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    kern<<<nunits, kda::simt::NT, smem, s>>>(
        static_cast<const TIn *>(q), static_cast<const TIn *>(k), static_cast<const TIn *>(v), g,
        beta, h0, hT, static_cast<TIn *>(o), T, H, hdr, cu, ntok, err);
    return launch_status();
}

template <typename TIn>
kda_status dispatch_simt(int D, const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *h0, float *hT, void *o, int T, int H,
                         int nunits, const int *hdr, const int *cu, long long ntok,
                         cudaStream_t s) {
    switch (D) {
        case 32:
            return launch_simt<32, TIn>(q, k, v, g, beta, h0, hT, o, T, H, nunits, hdr, cu, ntok, s);
        case 64:
            return launch_simt<64, TIn>(q, k, v, g, beta, h0, hT, o, T, H, nunits, hdr, cu, ntok, s);
        case 128:
            return launch_simt<128, TIn>(q, k, v, g, beta, h0, hT, o, T, H, nunits, hdr, cu, ntok,
                                         s);
        default: return KDA_ERR_UNSUPPORTED_SHAPE;
    }
}

// One state-pass launch over `units` units (chains * nseg); a.err_word and the
// test hook are filled in here.
template <int DVT>
kda_status launch_state(kda::tc::StateArgs a, long long units, cudaStream_t s) {
    using namespace kda::tc;
    const size_t smem = T5Layout<DVT>::BYTES;
    auto kern = kda_tc_state_kernel<DVT>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KDA_ERR_CUDA;
    a.err_word = device_error_word();
    if (!a.err_word) return KDA_ERR_CUDA;
    a.debug_drop_first_copy = debug_drop_first_copy();
    const long long grid = units * ((a.mode == kStateMap ? 2 * D : D) / DVT);
    if (grid > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    kern<<<(unsigned)grid, StateRoles<DVT>::THREADS, smem, s>>>(a);
    return launch_status();
}


// ---------------------------------------------------------------------------
// Backward pass.  Workspace: the forward path's header region (offsets check and
// chunk table of the packed layout), then the state checkpoints every bwd::CK
// tokens of every (sequence, head), then each CTA's scratch for the state every
// bwd::CB tokens of the chunk it is working on.
// ---------------------------------------------------------------------------
struct BwdLayout {
    size_t hdr_end, ckpt, sub, total;
};
BwdLayout bwd_layout(int B, int T, int H, int dk, int num_seqs, int dtype) {
    BwdLayout L{};
    const WsLayout F = ws_layout(B, T, H, dk, num_seqs, dtype, 1);
    L.hdr_end = F.recs;   // header, sequence offsets and chunk table only
    const long long ntok = (long long)B * T, N = num_seqs > 0 ? num_seqs : B;
    const long long slots = ntok / kda::bwd::CK + N + 1;
    L.ckpt = round_up(L.hdr_end, 256);
    L.sub = round_up(L.ckpt + (size_t)slots * H * dk * dk * sizeof(float), 256);
    L.total = L.sub + (size_t)N * H * kda::bwd::NSUB * dk * dk * sizeof(float);
    return L;
}

// Segmented backward (tensor-core path, fixed-length input): chains cut into segments of
// sc chunks, sc the smallest power of two dividing the chunks per sequence for which
// the segments number at most kBwdUnits (each unit holds the per-CTA scratch of
// NSUB states per slice, 512 KiB at d = 128); 0 when no cut leaves two segments.
constexpr long long kBwdUnits = 1024;
int bwd_seg_chunks(long long chains, int cps) {
    if (chains <= 0 || cps < 2) return 0;
    for (int sc = 1; sc < cps && cps % sc == 0; sc *= 2)
        if (chains * (cps / sc) <= kBwdUnits) return sc;
    return 0;
}
// Its workspace: the forward's (records), the reversed records, the states at the
// segment starts and the state gradients at the segment ends (nfw = floor(T / (sc C))
// slots per sequence each), then the per-token pass's checkpoints and scratch.
struct BwdSegLayout {
    WsLayout F;
    size_t rrec, fck, rck, ckpt, sub, total;
    int sc, nseg, nfw, cps;
};
// sc chunks per segment (sc divides the chunks per sequence, at least two segments);
// sc = 0: the policy above.  S.sc == 0 when no such cut exists.
BwdSegLayout bwd_seg_layout(int B, int T, int H, int dk, int dtype, int sc = 0) {
    BwdSegLayout S{};
    if (!is_tc_path(dtype, dk) || B <= 0 || T <= 0) return S;
    S.cps = (T + kda::tc::C - 1) / kda::tc::C;
    S.sc = sc > 0 ? (sc < S.cps && S.cps % sc == 0 ? sc : 0) : bwd_seg_chunks((long long)B * H, S.cps);
    if (!S.sc) return S;
    S.nseg = S.cps / S.sc;
    S.nfw = T / (S.sc * kda::tc::C);
    S.F = ws_layout(B, T, H, dk, 0, dtype, 1);
    S.rrec = round_up(S.F.total, 256);
    S.fck = round_up(S.rrec + (size_t)S.F.max_chunks * H * kda::tc::REC_BYTES, 256);
    const size_t states = (size_t)B * S.nfw * H * dk * dk * sizeof(float);
    S.rck = round_up(S.fck + states, 256);
    const long long slots = (long long)B * T / kda::bwd::CK + B + 1;
    S.ckpt = round_up(S.rck + states, 256);
    S.sub = round_up(S.ckpt + (size_t)slots * H * dk * dk * sizeof(float), 256);
    S.total = S.sub + (size_t)B * H * S.nseg * kda::bwd::NSUB * dk * dk * sizeof(float);
    return S;
}

template <int D, typename TIn>
kda_status launch_bwd(const void *q, const void *k, const void *v, const float *g,
                      const float *beta, const float *h0, const int32_t *cu, const int *hdr,
                      const void *dO, const float *dhT, int T, int H, long long ntok,
                      long long chains, float *ckpt, float *sub, void *dq, void *dkk, void *dvv,
                      float *dg, float *db, float *dh0, int *err, cudaStream_t s, int nseg = 1,
                      int seg_chunks = 1, const float *s_start = nullptr,
                      const float *g_end = nullptr, int nfw = 0, int cps = 0) {
    using namespace kda::bwd;
    const size_t smem = sizeof(BwdSmem<D, TIn>);
    auto kern = kda_bwd_slice_kernel<D, TIn>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KDA_ERR_CUDA;
    const long long grid = chains * nseg * (D / SLC);
    if (grid > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    // the D / SLC column slices of a chain (or of a segment of it) are one thread-block cluster
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(NTB);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = D / SLC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, static_cast<const TIn *>(q), static_cast<const TIn *>(k),
                           static_cast<const TIn *>(v), g, beta, h0, (const int *)cu, hdr,
                           static_cast<const TIn *>(dO), dhT, T, H, ckpt, sub,
                           static_cast<TIn *>(dq), static_cast<TIn *>(dkk),
                           static_cast<TIn *>(dvv), dg, db, dh0, ntok, err, nseg, seg_chunks,
                           s_start, g_end, nfw, cps) != cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    return launch_status();
}

}  // namespace

extern "C" {

int kda_version(void) { return 200; }

int kda_build_flags(void) { return KDA_DEBUG ? KDA_BUILD_DEBUG_CHECKS : 0; }

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null pointer, negative size or bad dtype";
        case KDA_ERR_UNSUPPORTED_SHAPE: return "KDA_ERR_UNSUPPORTED_SHAPE: need d_k == d_v in {32, 64, 128}";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: a pointer breaks its alignment rule (see kda.h)";
        case KDA_ERR_WORKSPACE_TOO_SMALL: return "KDA_ERR_WORKSPACE_TOO_SMALL";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA launch or query failed";
        case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
        case KDA_ERR_BAD_SEQLENS: return "KDA_ERR_BAD_SEQLENS: cu_seqlens not monotone or out of range";
        case KDA_ERR_EXCEEDS_STATIC_SCRATCH:
            return "KDA_ERR_EXCEEDS_STATIC_SCRATCH: problem needs more scratch than the 32 MiB "
                   "static array of kda_fwd_noalloc; use kda_fwd with a workspace";
        case KDA_ERR_CHECKPOINT_CAPACITY:
            return "KDA_ERR_CHECKPOINT_CAPACITY: the sequences have more state checkpoints than "
                   "ckpt_capacity slots";
        case KDA_ERR_BAD_ACCEPTED:
            return "KDA_ERR_BAD_ACCEPTED: an accepted token count of kda_decode_commit is outside "
                   "[0, K]; that sequence's state was left unchanged";
        case KDA_ERR_DEBUG_BOUNDS:
            return "KDA_ERR_DEBUG_BOUNDS: a device-side bounds check of the debug build failed; "
                   "the affected CTAs wrote nothing";
        default: return "KDA_ERR_UNKNOWN";
    }
}

size_t kda_fwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int dtype) {
    if (B < 0 || T < 0 || num_seqs < 0) return 0;
    if (check_shape(H, dk, dv, dtype) != KDA_OK) return 0;
    if (num_seqs > 0 && B != 1) return 0;
    return ws_layout(B, T, H, dk, num_seqs, dtype).total;
}

// Shared validation of the prefill entry points.  Fills N (the number of
// sequences) and the workspace layout.
static kda_status validate_fwd(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *h0, const int32_t *cu,
                               int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                               const void *o, const float *hT, const void *workspace,
                               size_t ws_bytes, bool need_inputs, bool need_outputs, int *N,
                               WsLayout *L, int nseg_req = 0) {
    if (B < 0 || T < 0 || num_seqs < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_shape(H, dk, dv, dtype);
    if (st != KDA_OK) return st;
    const bool varlen = cu != nullptr;
    if (varlen && (B != 1 || num_seqs <= 0)) return KDA_ERR_INVALID_ARG;
    if (!varlen && num_seqs != 0) return KDA_ERR_INVALID_ARG;
    *N = varlen ? num_seqs : B;
    const long long ntok = (long long)B * T;
    if (need_inputs && ntok > 0 && (!q || !k || !v || !g || !beta)) return KDA_ERR_INVALID_ARG;
    if (need_outputs && ntok > 0 && !o) return KDA_ERR_INVALID_ARG;
    // 16 B: rows staged with 16-byte copies; 8 B: float2 state access; else natural.
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    if (!aligned_to(q, 16) || !aligned_to(k, 16) || !aligned_to(v, 16) ||
        !aligned_to(workspace, 16) || !aligned_to(h0, 16) || !aligned_to(hT, 16) ||
        !aligned_to(g, 8) || !aligned_to(beta, 4) || !aligned_to(cu, 4) || !aligned_to(o, 2 * es))
        return KDA_ERR_MISALIGNED;
    // the tensor-core path loads g by tensor copies: a 16-byte aligned base
    if (is_tc_path(dtype, dk) && !aligned_to(g, 16)) return KDA_ERR_MISALIGNED;
    // outputs must not alias inputs (hT == h0 is the one allowed overlap)
    if (o && (o == q || o == k || o == v || o == g || o == beta)) return KDA_ERR_INVALID_ARG;
    if (nseg_req < 0 || nseg_req > kMaxSegmentsExplicit) return KDA_ERR_INVALID_ARG;
    if (nseg_req > 1 && !is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    *L = ws_layout(B, T, H, dk, varlen ? num_seqs : 0, dtype, nseg_req,
                   nseg_req > 0 ? kSplitSmBound : device_sms());
    if (!workspace || ws_bytes < L->total) return KDA_ERR_WORKSPACE_TOO_SMALL;
    if ((long long)(*N) * H * 8 > 0x7fffffffLL || L->max_chunks > 0x7fffffffLL)
        return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

// cuTensorMapEncodeTiled, reached through the runtime's driver entry points (no
// -lcuda); null if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// Tensor map of a [B, T, H, 128] input seen as the 4-D tensor (channel, head, token,
// sequence), innermost first: boxes of `box_c` channels x 1 head x `box_t` tokens x 1
// sequence.  bf16 inputs use 64-channel boxes with the 128-byte swizzle (the tensor
// core's K-major operand layout); fp32 g uses whole 512-byte rows without swizzle.
bool encode_input_map(CUtensorMap *m, const void *base, bool bf16, int H, long long T, int B,
                      int box_c, int box_t) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t es = bf16 ? 2 : 4, D = kda::tc::D;
    const cuuint64_t dims[4] = {D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {D * es, (cuuint64_t)H * D * es, (cuuint64_t)T * H * D * es};
    const cuuint32_t box[4] = {(cuuint32_t)box_c, 1, (cuuint32_t)box_t, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
               const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The prep's four input tensor maps: q, k, v as 64-channel x 64-token boxes, g as
// 32 whole rows.
static bool encode_inputs(const void *q, const void *k, const void *v, const float *g, int H, int T,
                   int nb, CUtensorMap *tq, CUtensorMap *tk, CUtensorMap *tv, CUtensorMap *tg) {
    using kda::tc::C;
    using kda::tc::D;
    return encode_input_map(tq, q, true, H, T, nb, 64, C) &&
           encode_input_map(tk, k, true, H, T, nb, 64, C) &&
           encode_input_map(tv, v, true, H, T, nb, 64, C) &&
           encode_input_map(tg, g, false, H, T, nb, D, C / 2);
}

// Tensor-core path, phase 1: chunk map (varlen) and the per-(chunk, head) records.
static kda_status tc_intra(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const int32_t *cu, int N, int T, int H,
                           const WsLayout &L, void *workspace, cudaStream_t s) {
    using namespace kda::tc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *hdr = reinterpret_cast<int *>(ws + L.hdr);
    int *seq_off = reinterpret_cast<int *>(ws + L.seq_off);
    auto *chunks = reinterpret_cast<ChunkLoc *>(ws + L.chunks);
    kda_status st;
    int cps = 0;
    if (cu) {
        int *err = device_error_word();
        if (!err) return KDA_ERR_CUDA;
        kda_chunk_map_kernel<<<1, 1024, 0, s>>>(cu, N, T, hdr, seq_off, chunks,
                                                (int)L.max_chunks, err, ERRBIT_SEQLENS);
        if ((st = launch_status()) != KDA_OK) return st;
    } else {
        cps = (T + C - 1) / C;
    }
    if (L.max_chunks == 0) return KDA_OK;
    const size_t smem = sizeof(PrepSmem) + 1024;   // + slack for 1024-byte alignment
    if (cudaFuncSetAttribute(kda_tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return KDA_ERR_CUDA;
    // persistent: two CTAs per SM (the kernel's shared memory allows no more), each
    // walking the (chunk, head) items with a stride of the grid
    const long long items = L.max_chunks * H;
    if (items > 0x7fffffffLL - 4096) return KDA_ERR_INVALID_ARG;   // int item indices
    const int sms = device_sms();
    const long long cap = 2LL * (sms > 0 ? sms : 148);
    const unsigned grid = (unsigned)(items < cap ? items : cap);
    // inputs as (channel, head, token, sequence); packed sequences are one long sequence
    // whose per-chunk bounds the kernel applies itself
    const int nb = cu ? 1 : N;
    CUtensorMap tq, tk, tv, tg;
    if (!encode_inputs(q, k, v, g, H, T, nb, &tq, &tk, &tv, &tg)) return KDA_ERR_CUDA;
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    PrepArgs p{};
    p.beta = beta;
    p.T = T;
    p.H = H;
    p.cps = cps;
    p.slots = (int)L.max_chunks;
    p.hdr = hdr;
    p.chunks = cu ? chunks : nullptr;
    p.recs = ws + L.recs;
    p.err_word = err;
    p.nseq = N;
    kda_tc_prep_kernel<<<grid, kPrepThreads, smem, s>>>(tq, tk, tv, tg, p);
    return launch_status();
}

// The state pass's arguments for an output pass over the records (no T-split).
static kda::tc::StateArgs state_args(const float *h0, const int32_t *cu, int N, int T, int H,
                                     const WsLayout &L, void *o, float *hT, void *workspace,
                                     float *ckpt, int ckpt_chunks, long long ckpt_cap) {
    using namespace kda::tc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    StateArgs a{};
    a.recs = ws + L.recs;
    a.h0 = h0;
    a.hT = hT;
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.T = T;
    a.H = H;
    a.cps = cu ? 0 : (T + C - 1) / C;
    a.hdr = reinterpret_cast<int *>(ws + L.hdr);
    a.seq_off = reinterpret_cast<int *>(ws + L.seq_off);
    a.cu = cu;
    a.nseg = 1;
    a.mode = kStateOutput;
    a.ckpt = ckpt;
    a.ckpt_chunks = ckpt_chunks;
    a.ckpt_cap = ckpt_cap;
    a.ntok = cu ? (long long)T : (long long)N * T;
    a.max_chunks = (int)L.max_chunks;
    return a;
}

// Tensor-core path, phase 2: the state pass over the records.
static kda_status tc_inter(const float *h0, const int32_t *cu, int N, int T, int H,
                           const WsLayout &L, void *o, float *hT, void *workspace,
                           cudaStream_t s, float *ckpt = nullptr, int ckpt_chunks = 0,
                           long long ckpt_cap = 0) {
    using namespace kda::tc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *hdr = reinterpret_cast<int *>(ws + L.hdr);
    StateArgs a = state_args(h0, cu, N, T, H, L, o, hT, workspace, ckpt, ckpt_chunks, ckpt_cap);
    a.nseg = L.nseg;
    const long long chains = (long long)N * H;
    if (L.nseg <= 1) {
        // 32-column slices give the shortest per-chunk latency (they suit few chains);
        // with more than two waves of them the pass is throughput-bound and 64-column
        // slices (half the CTAs, each chunk's map read once per two slices) are faster
        const int sms = device_sms();
        if (chains * (D / 32) > 2LL * (sms > 0 ? sms : 148)) return launch_state<64>(a, chains, s);
        return launch_state<32>(a, chains, s);
    }
    // T-split: segment maps, the sequential combine, then the output pass from
    // each segment's true starting state.
    float *s_in = reinterpret_cast<float *>(ws + L.s_in);
    float *seg_map = reinterpret_cast<float *>(ws + L.seg_map);
    StateArgs m = a;
    m.mode = kStateMap;
    m.seg_map = seg_map;
    kda_status st = launch_state<32>(m, chains * L.nseg, s);
    if (st != KDA_OK) return st;
    if (chains > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    kda_tc_seg_combine_kernel<<<dim3((unsigned)chains, D / 32), 256, 0, s>>>(
        h0, seg_map, s_in, L.nseg, hdr, cu ? 1 : 0);
    if ((st = launch_status()) != KDA_OK) return st;
    a.s_in = s_in;
    return launch_state<32>(a, chains * L.nseg, s);
}

// Overlapped schedule (kda_tc_fused_kernel): one block per SM, 2 state CTAs
// (64-column slices) per chain and two prep workers in every other block.  Chosen by
// kda_fwd for fixed-length input without a T-split when its estimated time beats the
// two launches by 5%.  The estimates use per-unit times measured on a B200 (1,965 MHz):
//   two launches: a prep item takes a worker 12.2 us with 2 workers on every SM, then
//     the 32-column state pass takes 0.79 us per chunk per wave of 4 CTAs per chain;
//   one launch: a prep item takes 14.5 us (it shares the GPU with the state pass), a
//     64-column chunk 1.19 us, and the chain starts about 5 us after the launch.
// Below 128 chunks per chain the two were measured equal or the single launch slower
// (B=2, H=8, T=4,096: 0.110 against 0.107 ms), so the single launch needs at least that
// many (B=1, H=16, T=16,384: 0.380 against 0.416 ms; T=1M: 19.5 against 23.8 ms).
// The constants were fitted before the state pass had a producer warp per ring and the
// record window its 32 MiB (one launch at T=1M: 15.9 against 22.5 ms now; a 64-column
// chunk about 0.93 us inside it): the model errs toward the two launches, and picks the
// single launch for about 12 or more chains, where it was measured faster.
constexpr double kPrepUsTwo = 12.2, kState32Us = 0.79;
constexpr double kPrepUsOne = 14.5, kState64OneUs = 1.19, kRampUs = 5.0;
constexpr long long kMinOverlapChunks = 128;
static bool overlap_schedule(long long chains, long long cps, int sms) {
    if (chains <= 0 || cps < kMinOverlapChunks || sms <= 0) return false;
    const long long nstate = 2 * chains;
    if (nstate > sms / 2) return false;
    const double c = (double)chains, n = (double)cps;
    const double prep_one = c * kPrepUsOne / (2.0 * (double)(sms - nstate));
    const double one = n * (prep_one > kState64OneUs ? prep_one : kState64OneUs) + kRampUs;
    const double two = n * (c * kPrepUsTwo / (2.0 * sms) +
                            kState32Us * (double)((4 * chains + sms - 1) / sms));
    return one < 0.95 * two;
}

// Both phases as one launch (fixed-length input, no T-split).  *refused is set when
// the launch itself was refused (e.g. the device cannot hold one such block per SM
// at once), with nothing started, so the caller may take the two launches instead.
static kda_status tc_fused(bool *refused, const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, int N, int T, int H,
                           const WsLayout &L, void *o, float *hT, void *workspace,
                           cudaStream_t s, float *ckpt = nullptr, int ckpt_chunks = 0,
                           long long ckpt_cap = 0) {
    using namespace kda::tc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const long long chains = (long long)N * H, items = L.max_chunks * H;
    if (items == 0 || items > 0x7fffffffLL - 4096) return KDA_ERR_INVALID_ARG;
    const int sms = device_sms();
    if (sms <= 0) return KDA_ERR_CUDA;
    const long long nstate = 2 * chains;   // 64-column slices
    if (nstate >= sms) return KDA_ERR_INVALID_ARG;
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    CUtensorMap tq, tk, tv, tg;
    if (!encode_inputs(q, k, v, g, H, T, N, &tq, &tk, &tv, &tg)) return KDA_ERR_CUDA;
    int *ready = reinterpret_cast<int *>(ws + L.ready);
    int *prog = reinterpret_cast<int *>(ws + L.prog);
    if (nstate > kProgressSlots) return KDA_ERR_INVALID_ARG;
    // flags and counters are contiguous: one memset
    if (cudaMemsetAsync(ready, 0, L.prog + kProgressSlots * kProgStride * sizeof(int) - L.ready, s) !=
        cudaSuccess) {
        cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    PrepArgs p{};
    p.beta = beta;
    p.T = T;
    p.H = H;
    p.cps = (T + C - 1) / C;
    p.slots = (int)L.max_chunks;
    p.hdr = reinterpret_cast<int *>(ws + L.hdr);
    p.chunks = nullptr;
    p.recs = ws + L.recs;
    p.err_word = err;
    p.ready = ready;
    p.nseq = N;
    p.nstate = (int)nstate;
    p.progress = prog;
    // records in flight between the roles: about 32 MiB, well inside L2 (B=1, H=16,
    // T=1M: 21 chunks per chain; measured 16.2 ms at 20 chunks, 16.7 at 31, 17.9 at 40)
    const long long win = (32LL << 20) / (chains * (long long)REC_BYTES);
    p.window = (int)(win < 2 ? 2 : win);
    StateArgs a = state_args(h0, nullptr, N, T, H, L, o, hT, workspace, ckpt, ckpt_chunks, ckpt_cap);
    a.err_word = err;
    a.debug_drop_first_copy = debug_drop_first_copy();
    a.ready = ready;
    a.progress = prog;
    if (cudaFuncSetAttribute(kda_tc_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kFusedSmem) != cudaSuccess) {
        cudaGetLastError();
        if (refused) *refused = true;
        return KDA_ERR_CUDA;
    }
    // every block must be resident at once (state blocks wait for prep blocks): one
    // block per SM, launched cooperatively
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(kFusedThreads);
    cfg.dynamicSmemBytes = kFusedSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kda_tc_fused_kernel, tq, tk, tv, tg, p, a, (int)nstate) !=
        cudaSuccess) {
        cudaGetLastError();
        if (refused) *refused = true;
        return KDA_ERR_CUDA;
    }
    return launch_status();
}

// Whether kda_fwd takes the overlapped schedule for this problem.
static bool use_overlap(const int32_t *cu, int N, int T, int H, const WsLayout &L) {
    if (cu || L.nseg > 1 || T <= 0) return false;
    return overlap_schedule((long long)N * H, ((long long)T + kda::tc::C - 1) / kda::tc::C,
                            device_sms());
}

kda_status kda_fwd_intra(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const int32_t *cu_seqlens, int num_seqs, int B,
                         int T, int H, int dk, int dv, int dtype, void *workspace,
                         size_t ws_bytes, void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, nullptr, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, nullptr, nullptr, workspace, ws_bytes, true, false, &N, &L);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return KDA_OK;
    return tc_intra(q, k, v, g, beta, cu_seqlens, N, T, H, L, workspace,
                    static_cast<cudaStream_t>(stream));
}

kda_status kda_fwd_inter(const float *h0, const int32_t *cu_seqlens, int num_seqs, int B, int T,
                         int H, int dk, int dv, int dtype, void *o, float *hT, void *workspace,
                         size_t ws_bytes, void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, h0, cu_seqlens,
                                 num_seqs, B, T, H, dk, dv, dtype, o, hT, workspace, ws_bytes,
                                 false, true, &N, &L);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return KDA_OK;
    return tc_inter(h0, cu_seqlens, N, T, H, L, o, hT, workspace,
                    static_cast<cudaStream_t>(stream));
}

kda_status kda_fwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                   int B, int T, int H, int dk, int dv, int dtype, void *o, float *hT,
                   void *workspace, size_t ws_bytes, void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, o, hT, workspace, ws_bytes, true, true, &N, &L);
    if (st != KDA_OK) return st;
    if (N == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (is_tc_path(dtype, dk)) {
        if (use_overlap(cu_seqlens, N, T, H, L)) {
            bool refused = false;
            st = tc_fused(&refused, q, k, v, g, beta, h0, N, T, H, L, o, hT, workspace, s);
            if (!refused) return st;   // else: the two launches below
        }
        if ((st = tc_intra(q, k, v, g, beta, cu_seqlens, N, T, H, L, workspace, s)) != KDA_OK)
            return st;
        return tc_inter(h0, cu_seqlens, N, T, H, L, o, hT, workspace, s);
    }
    // fp32 / small-head path
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *hdr = reinterpret_cast<int *>(ws + L.hdr);
    if (cu_seqlens) {
        int *err = device_error_word();
        if (!err) return KDA_ERR_CUDA;
        kda::tc::kda_chunk_map_kernel<<<1, 1024, 0, s>>>(
            cu_seqlens, N, T, hdr, reinterpret_cast<int *>(ws + L.seq_off),
            reinterpret_cast<kda::tc::ChunkLoc *>(ws + L.chunks), (int)L.max_chunks, err,
            ERRBIT_SEQLENS);
        if ((st = launch_status()) != KDA_OK) return st;
    }
    const int nunits = N * H;
    const long long ntok = (long long)B * T;
    if (dtype == KDA_DTYPE_F32)
        return dispatch_simt<float>(dk, q, k, v, g, beta, h0, hT, o, T, H, nunits, hdr,
                                    cu_seqlens, ntok, s);
    return dispatch_simt<__nv_bfloat16>(dk, q, k, v, g, beta, h0, hT, o, T, H, nunits, hdr,
                                        cu_seqlens, ntok, s);
}

kda_status kda_fwd_checkpointed(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *h0, const int32_t *cu_seqlens,
                                int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                                void *o, float *hT, int ckpt_every, float *ckpts,
                                long long ckpt_capacity, void *workspace, size_t ws_bytes,
                                void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, o, hT, workspace, ws_bytes, true, true, &N, &L);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (ckpt_every <= 0 || ckpt_every % kda::tc::C != 0 || ckpt_capacity < 0)
        return KDA_ERR_INVALID_ARG;
    if (ckpt_capacity > 0 && !ckpts) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(ckpts, 16)) return KDA_ERR_MISALIGNED;
    if (!cu_seqlens && (long long)B * (T / ckpt_every) > ckpt_capacity) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_overlap(cu_seqlens, N, T, H, L)) {
        bool refused = false;
        st = tc_fused(&refused, q, k, v, g, beta, h0, N, T, H, L, o, hT, workspace, s, ckpts,
                      ckpt_every / kda::tc::C, ckpt_capacity);
        if (!refused) return st;   // else: the two launches below
    }
    if ((st = tc_intra(q, k, v, g, beta, cu_seqlens, N, T, H, L, workspace, s)) != KDA_OK)
        return st;
    return tc_inter(h0, cu_seqlens, N, T, H, L, o, hT, workspace, s, ckpts,
                    ckpt_every / kda::tc::C, ckpt_capacity);
}

int kda_fwd_plan_overlap(int B, int T, int H, int dk, int dv, int num_seqs, int dtype) {
    if (B < 0 || T < 0 || num_seqs != 0) return 0;
    if (check_shape(H, dk, dv, dtype) != KDA_OK || !is_tc_path(dtype, dk)) return 0;
    const WsLayout L = ws_layout(B, T, H, dk, 0, dtype, 0, device_sms());
    return use_overlap(nullptr, B, T, H, L) ? 1 : 0;
}

kda_status kda_fwd_overlapped(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *h0, int B, int T, int H, int dk,
                              int dv, int dtype, void *o, float *hT, void *workspace,
                              size_t ws_bytes, void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, h0, nullptr, 0, B, T, H, dk, dv, dtype, o, hT,
                                 workspace, ws_bytes, true, true, &N, &L, /*nseg_req=*/1);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    const int sms = device_sms();
    if (sms <= 0) return KDA_ERR_CUDA;
    if (2LL * N * H >= sms) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (N == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) return tc_inter(h0, nullptr, N, T, H, L, o, hT, workspace, s);   // hT = h0
    return tc_fused(nullptr, q, k, v, g, beta, h0, N, T, H, L, o, hT, workspace, s);
}

int kda_fwd_plan_segments(int B, int T, int H, int dk, int dv, int num_seqs, int dtype) {
    if (B < 0 || T < 0 || num_seqs < 0) return 0;
    if (check_shape(H, dk, dv, dtype) != KDA_OK) return 0;
    if (num_seqs > 0 && B != 1) return 0;
    return ws_layout(B, T, H, dk, num_seqs, dtype, 0, device_sms()).nseg;
}

size_t kda_fwd_segmented_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                        int dtype, int num_segments) {
    if (B < 0 || T < 0 || num_seqs < 0) return 0;
    if (num_segments < 1 || num_segments > kMaxSegmentsExplicit) return 0;
    if (check_shape(H, dk, dv, dtype) != KDA_OK) return 0;
    if (num_seqs > 0 && B != 1) return 0;
    if (num_segments > 1 && !is_tc_path(dtype, dk)) return 0;
    return ws_layout(B, T, H, dk, num_seqs, dtype, num_segments).total;
}

kda_status kda_fwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                             int num_segments, void *o, float *hT, void *workspace,
                             size_t ws_bytes, void *stream) {
    if (num_segments < 1) return KDA_ERR_INVALID_ARG;
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, o, hT, workspace, ws_bytes, true, true, &N, &L,
                                 num_segments);
    if (st != KDA_OK) return st;
    if (N == 0) return KDA_OK;
    if (!is_tc_path(dtype, dk))   // num_segments == 1 here: the plain pass
        return kda_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv, dtype, o, hT,
                       workspace, ws_bytes, stream);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = tc_intra(q, k, v, g, beta, cu_seqlens, N, T, H, L, workspace, s)) != KDA_OK)
        return st;
    return tc_inter(h0, cu_seqlens, N, T, H, L, o, hT, workspace, s);
}

kda_status kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, float *S, void *o, int N, int H, int dk, int dv,
                           int dtype, void *stream) {
    if (N < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_shape(H, dk, dv, dtype);
    if (st != KDA_OK) return st;
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !g || !beta || !S || !o) return KDA_ERR_INVALID_ARG;
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    if (!aligned_to(S, 16) || !aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) ||
        !aligned_to(o, es) || !aligned_to(g, 4) || !aligned_to(beta, 4))
        return KDA_ERR_MISALIGNED;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)(N * H);
    using namespace kda::dec;
#define KDA_DEC(DD, TT)                                                                       \
    kda_decode_kernel<DD, TT><<<grid, NT, 0, s>>>(                                            \
        static_cast<const TT *>(q), static_cast<const TT *>(k), static_cast<const TT *>(v), g, \
        beta, S, static_cast<TT *>(o))
    if (dtype == KDA_DTYPE_BF16) {
        if (dk == 32) KDA_DEC(32, __nv_bfloat16);
        else if (dk == 64) KDA_DEC(64, __nv_bfloat16);
        else KDA_DEC(128, __nv_bfloat16);
    } else {
        if (dk == 32) KDA_DEC(32, float);
        else if (dk == 64) KDA_DEC(64, float);
        else KDA_DEC(128, float);
    }
#undef KDA_DEC
    return launch_status();
}

// Shared host checks of the verify / commit entry points.
static kda_status check_multi(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const float *S, int N, int K, int H, int dk,
                              int dv, int dtype, bool need_q) {
    if (N < 0 || K < 0) return KDA_ERR_INVALID_ARG;
    kda_status st = check_shape(H, dk, dv, dtype);
    if (st != KDA_OK) return st;
    if (K > kda::dec::kMaxDraft) return KDA_ERR_INVALID_ARG;
    if (N == 0 || K == 0) return KDA_OK;
    if ((need_q && !q) || !k || !v || !g || !beta || !S) return KDA_ERR_INVALID_ARG;
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    if (!aligned_to(S, 16) || !aligned_to(q, es) || !aligned_to(k, es) || !aligned_to(v, es) ||
        !aligned_to(g, 4) || !aligned_to(beta, 4))
        return KDA_ERR_MISALIGNED;
    if ((long long)N * H > 0x7fffffffLL || (long long)N * K * H > 0x7fffffffLL)
        return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

kda_status kda_decode_verify(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *S, void *o, int N, int K, int H,
                             int dk, int dv, int dtype, void *stream) {
    kda_status st = check_multi(q, k, v, g, beta, S, N, K, H, dk, dv, dtype, true);
    if (st != KDA_OK) return st;
    if (N == 0 || K == 0) return KDA_OK;
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    if (!o) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(o, es)) return KDA_ERR_MISALIGNED;
    if (o == q || o == k || o == v || o == g || o == beta || o == S) return KDA_ERR_INVALID_ARG;
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)(N * H);
    using namespace kda::dec;
#define KDA_VER(DD, TT)                                                                         \
    kda_decode_multi_kernel<DD, TT, false><<<grid, NT, 0, s>>>(                                 \
        static_cast<const TT *>(q), static_cast<const TT *>(k), static_cast<const TT *>(v), g,   \
        beta, const_cast<float *>(S), static_cast<TT *>(o), nullptr, K, H, err)
    if (dtype == KDA_DTYPE_BF16) {
        if (dk == 32) KDA_VER(32, __nv_bfloat16);
        else if (dk == 64) KDA_VER(64, __nv_bfloat16);
        else KDA_VER(128, __nv_bfloat16);
    } else {
        if (dk == 32) KDA_VER(32, float);
        else if (dk == 64) KDA_VER(64, float);
        else KDA_VER(128, float);
    }
#undef KDA_VER
    return launch_status();
}

kda_status kda_decode_commit(const void *k, const void *v, const float *g, const float *beta,
                             const int32_t *accepted, float *S, int N, int K, int H, int dk,
                             int dv, int dtype, void *stream) {
    kda_status st = check_multi(nullptr, k, v, g, beta, S, N, K, H, dk, dv, dtype, false);
    if (st != KDA_OK) return st;
    if (N == 0 || K == 0) return KDA_OK;
    if (!accepted) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(accepted, 4)) return KDA_ERR_MISALIGNED;
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)(N * H);
    using namespace kda::dec;
#define KDA_COM(DD, TT)                                                                         \
    kda_decode_multi_kernel<DD, TT, true><<<grid, NT, 0, s>>>(                                  \
        nullptr, static_cast<const TT *>(k), static_cast<const TT *>(v), g, beta, S, nullptr,    \
        accepted, K, H, err)
    if (dtype == KDA_DTYPE_BF16) {
        if (dk == 32) KDA_COM(32, __nv_bfloat16);
        else if (dk == 64) KDA_COM(64, __nv_bfloat16);
        else KDA_COM(128, __nv_bfloat16);
    } else {
        if (dk == 32) KDA_COM(32, float);
        else if (dk == 64) KDA_COM(64, float);
        else KDA_COM(128, float);
    }
#undef KDA_COM
    return launch_status();
}

size_t kda_bwd_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs, int dtype) {
    return kda_bwd_segmented_workspace_size(B, T, H, dk, dv, num_seqs, dtype, 0);
}

int kda_bwd_plan_segments(int B, int T, int H, int dk, int dv, int num_seqs, int dtype) {
    if (B < 0 || T < 0 || num_seqs < 0 || check_shape(H, dk, dv, dtype) != KDA_OK) return 0;
    if (num_seqs > 0) return 1;
    const BwdSegLayout S = bwd_seg_layout(B, T, H, dk, dtype);
    return S.sc ? S.nseg : 1;
}

// num_segments == 0: kda_bwd's choice; 1: the per-chain pass; n >= 2: n segments.
size_t kda_bwd_segmented_workspace_size(int B, int T, int H, int dk, int dv, int num_seqs,
                                        int dtype, int num_segments) {
    if (B < 0 || T < 0 || num_seqs < 0 || num_segments < 0) return 0;
    if (check_shape(H, dk, dv, dtype) != KDA_OK) return 0;
    if (num_seqs > 0 && B != 1) return 0;
    const size_t old = bwd_layout(B, T, H, dk, num_seqs, dtype).total;
    if (num_segments == 1) return old;
    if (num_segments >= 2) {
        if (num_seqs > 0 || T <= 0) return 0;
        const int cps = (T + kda::tc::C - 1) / kda::tc::C;
        if (cps % num_segments) return 0;
        return bwd_seg_layout(B, T, H, dk, dtype, cps / num_segments).total;
    }
    const size_t seg = num_seqs > 0 ? 0 : bwd_seg_layout(B, T, H, dk, dtype).total;
    return old > seg ? old : seg;
}

// nseg_req: 0 the policy, 1 the per-chain pass, n >= 2 n segments.
static kda_status bwd_impl(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, const int32_t *cu_seqlens,
                           int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                           const void *grad_o, const float *grad_hT, void *grad_q, void *grad_k,
                           void *grad_v, float *grad_g, float *grad_beta, float *grad_h0,
                           void *workspace, size_t ws_bytes, void *stream, int nseg_req) {
    if (nseg_req < 0) return KDA_ERR_INVALID_ARG;
    int N;
    WsLayout F;
    // the forward's checks cover the inputs; the outputs are checked here
    kda_status st = validate_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, grad_q, grad_h0, reinterpret_cast<void *>(uintptr_t(256)),
                                 SIZE_MAX, true, false, &N, &F, 1);
    if (st != KDA_OK) return st;
    const long long ntok = (long long)B * T;
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    if (ntok > 0 && (!grad_o || !grad_q || !grad_k || !grad_v || !grad_g || !grad_beta))
        return KDA_ERR_INVALID_ARG;
    // the slice kernel stages rows of g and grad_o with 16-byte copies
    if (!aligned_to(grad_o, 16) || !aligned_to(g, 16) || !aligned_to(grad_q, es) ||
        !aligned_to(grad_k, es) || !aligned_to(grad_v, es) || !aligned_to(grad_g, 4) ||
        !aligned_to(grad_beta, 4) || !aligned_to(grad_hT, 16) || !aligned_to(grad_h0, 16))
        return KDA_ERR_MISALIGNED;
    const void *ins[] = {q, k, v, g, beta, h0, grad_o, grad_hT};
    const void *outs[] = {grad_q, grad_k, grad_v, grad_g, grad_beta, grad_h0};
    for (const void *o : outs)
        for (const void *i : ins)
            if (o && o == i) return KDA_ERR_INVALID_ARG;
    const BwdLayout L = bwd_layout(B, T, H, dk, cu_seqlens ? num_seqs : 0, dtype);
    BwdSegLayout SL{};
    if (nseg_req >= 2) {   // explicit segments: tensor-core path, fixed length, n | chunks
        const int cps = (T + kda::tc::C - 1) / kda::tc::C;
        if (!cu_seqlens && T > 0 && cps % nseg_req == 0)
            SL = bwd_seg_layout(B, T, H, dk, dtype, cps / nseg_req);
        if (!SL.sc) return KDA_ERR_UNSUPPORTED_SHAPE;
        if (!aligned_to(grad_q, 16) || !aligned_to(grad_k, 16)) return KDA_ERR_MISALIGNED;
    } else if (nseg_req == 0 && !cu_seqlens) {
        SL = bwd_seg_layout(B, T, H, dk, dtype);
    }
    if (!workspace || ws_bytes < (L.total > SL.total ? L.total : SL.total))
        return KDA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned_to(workspace, 16)) return KDA_ERR_MISALIGNED;
    if (N == 0 || ntok == 0 && !grad_h0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *hdr = reinterpret_cast<int *>(ws + F.hdr);
    int *err = device_error_word();
    if (!err) return KDA_ERR_CUDA;
    if (cu_seqlens) {   // offsets check (the chunk table it also writes is not used here)
        kda::tc::kda_chunk_map_kernel<<<1, 1024, 0, s>>>(
            cu_seqlens, N, T, hdr, reinterpret_cast<int *>(ws + F.seq_off),
            reinterpret_cast<kda::tc::ChunkLoc *>(ws + F.chunks), (int)F.max_chunks, err,
            ERRBIT_SEQLENS);
        if ((st = launch_status()) != KDA_OK) return st;
    }
    const long long chains = (long long)N * H;
    // Segmented: the tensor-core forward with the state at every segment start (its o
    // goes to grad_q), the reversed records, the chunk-level gradient chain over them
    // from dL/dhT with dL/dS at every segment end (its o goes to grad_k), then the
    // per-token backward on all segments at once, which overwrites grad_q and grad_k.
    // 16-byte vector stores of grad_q and grad_k (the state passes' o); else the
    // per-chain pass.
    if (SL.sc && aligned_to(grad_q, 16) && aligned_to(grad_k, 16)) {
        using namespace kda::bwd;
        float *fck = reinterpret_cast<float *>(ws + SL.fck);
        float *rck = reinterpret_cast<float *>(ws + SL.rck);
        const long long nck_slots = (long long)N * SL.nfw;
        if ((st = tc_intra(q, k, v, g, beta, nullptr, N, T, H, SL.F, workspace, s)) != KDA_OK)
            return st;
        if ((st = tc_inter(h0, nullptr, N, T, H, SL.F, grad_q, nullptr, workspace, s, fck, SL.sc,
                           nck_slots)) != KDA_OK)
            return st;
        const size_t rsmem = sizeof(RevSmem);
        if (cudaFuncSetAttribute(kda_bwd_rev_records_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem) != cudaSuccess)
            return KDA_ERR_CUDA;
        const long long items = SL.F.max_chunks * H;
        const int sms = device_sms();
        const long long cap = 3LL * (sms > 0 ? sms : 148);
        kda_bwd_rev_records_kernel<<<(unsigned)(items < cap ? items : cap), kRevThreads, rsmem, s>>>(
            ws + SL.F.recs, static_cast<const __nv_bfloat16 *>(grad_o), ws + SL.rrec, T, H, SL.cps,
            items);
        if ((st = launch_status()) != KDA_OK) return st;
        WsLayout R = SL.F;
        R.recs = SL.rrec;
        if ((st = tc_inter(grad_hT, nullptr, N, T, H, R, grad_k, nullptr, workspace, s, rck, SL.sc,
                           nck_slots)) != KDA_OK)
            return st;
        return launch_bwd<128, __nv_bfloat16>(
            q, k, v, g, beta, h0, nullptr, hdr, grad_o, grad_hT, T, H, ntok, chains,
            reinterpret_cast<float *>(ws + SL.ckpt), reinterpret_cast<float *>(ws + SL.sub), grad_q,
            grad_k, grad_v, grad_g, grad_beta, grad_h0, err, s, SL.nseg, SL.sc, fck, rck, SL.nfw,
            SL.cps);
    }
    float *ckpt = reinterpret_cast<float *>(ws + L.ckpt);
    float *sub = reinterpret_cast<float *>(ws + L.sub);
#define KDA_BWD(DD, TT)                                                                    \
    return launch_bwd<DD, TT>(q, k, v, g, beta, h0, cu_seqlens, hdr, grad_o, grad_hT, T, H, \
                              ntok, chains, ckpt, sub, grad_q, grad_k, grad_v, grad_g,      \
                              grad_beta, grad_h0, err, s)
    if (dtype == KDA_DTYPE_BF16) {
        if (dk == 32) KDA_BWD(32, __nv_bfloat16);
        if (dk == 64) KDA_BWD(64, __nv_bfloat16);
        KDA_BWD(128, __nv_bfloat16);
    }
    if (dk == 32) KDA_BWD(32, float);
    if (dk == 64) KDA_BWD(64, float);
    KDA_BWD(128, float);
#undef KDA_BWD
}

kda_status kda_bwd(const void *q, const void *k, const void *v, const float *g,
                   const float *beta, const float *h0, const int32_t *cu_seqlens, int num_seqs,
                   int B, int T, int H, int dk, int dv, int dtype, const void *grad_o,
                   const float *grad_hT, void *grad_q, void *grad_k, void *grad_v,
                   float *grad_g, float *grad_beta, float *grad_h0, void *workspace,
                   size_t ws_bytes, void *stream) {
    return bwd_impl(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv, dtype, grad_o,
                    grad_hT, grad_q, grad_k, grad_v, grad_g, grad_beta, grad_h0, workspace,
                    ws_bytes, stream, 0);
}

kda_status kda_bwd_segmented(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *h0, const int32_t *cu_seqlens,
                             int num_seqs, int B, int T, int H, int dk, int dv, int dtype,
                             const void *grad_o, const float *grad_hT, void *grad_q, void *grad_k,
                             void *grad_v, float *grad_g, float *grad_beta, float *grad_h0,
                             int num_segments, void *workspace, size_t ws_bytes, void *stream) {
    return bwd_impl(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv, dtype, grad_o,
                    grad_hT, grad_q, grad_k, grad_v, grad_g, grad_beta, grad_h0, workspace,
                    ws_bytes, stream, num_segments);
}

// ---------------------------------------------------------------------------
// Context parallelism across devices (fixed-length input, tensor-core path).
// ---------------------------------------------------------------------------
size_t kda_cp_workspace_size(int B, int T_local, int H, int dk, int dv, int dtype) {
    if (!is_tc_path(dtype, dk) || dk != dv) return 0;
    return kda_fwd_segmented_workspace_size(B, T_local, H, dk, dv, 0, dtype, 1);
}

kda_status kda_cp_local_map(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, int B, int T_local, int H, int dk, int dv,
                            int dtype, float *seg_map, void *workspace, size_t ws_bytes,
                            void *stream) {
    int N;
    WsLayout L;
    kda_status st = validate_fwd(q, k, v, g, beta, nullptr, nullptr, 0, B, T_local, H, dk, dv,
                                 dtype, nullptr, nullptr, workspace, ws_bytes, true, false, &N,
                                 &L, 1);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (N > 0 && !seg_map) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(seg_map, 16)) return KDA_ERR_MISALIGNED;
    if (N == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = tc_intra(q, k, v, g, beta, nullptr, N, T_local, H, L, workspace, s)) != KDA_OK)
        return st;
    // the map pass over the whole local segment: [R | P] per (sequence, head)
    using namespace kda::tc;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    StateArgs m{};
    m.recs = ws + L.recs;
    m.T = T_local;
    m.H = H;
    m.cps = (T_local + C - 1) / C;
    m.hdr = reinterpret_cast<int *>(ws + L.hdr);
    m.seq_off = reinterpret_cast<int *>(ws + L.seq_off);
    m.nseg = 1;
    m.mode = kStateMap;
    m.seg_map = seg_map;
    m.ntok = (long long)N * T_local;
    m.max_chunks = (int)L.max_chunks;
    return launch_state<32>(m, (long long)N * H, s);
}

kda_status kda_cp_finish(const float *maps, int rank, int world, const float *h0, float *s_in,
                         int B, int T_local, int H, int dk, int dv, int dtype, void *o,
                         float *hT, void *workspace, size_t ws_bytes, void *stream) {
    if (world < 1 || rank < 0 || rank >= world) return KDA_ERR_INVALID_ARG;
    if (rank > 0 && !maps) return KDA_ERR_INVALID_ARG;
    int N;
    WsLayout L;
    kda_status st = validate_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, h0, nullptr, 0, B,
                                 T_local, H, dk, dv, dtype, o, hT, workspace, ws_bytes, false,
                                 true, &N, &L, 1);
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (N > 0 && !s_in) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(maps, 16) || !aligned_to(s_in, 16)) return KDA_ERR_MISALIGNED;
    if (s_in == h0 || s_in == hT || (const void *)s_in == o) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long chains = (long long)N * H;
    if (chains > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    kda::tc::kda_cp_combine_kernel<<<dim3((unsigned)chains, kda::tc::D / 32), 256, 0, s>>>(
        h0, maps, s_in, rank, (int)chains);
    if ((st = launch_status()) != KDA_OK) return st;
    return tc_inter(s_in, nullptr, N, T_local, H, L, o, hT, workspace, s);
}

kda_status kda_get_last_device_error(void *stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_kda_device_error, sizeof(int)) != cudaSuccess)
        return KDA_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_kda_device_error, &zero, sizeof(int)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word & ERRBIT_SEQLENS) return KDA_ERR_BAD_SEQLENS;
    if (word & ERRBIT_TIMEOUT) return KDA_ERR_DEVICE_TIMEOUT;
    if (word & ERRBIT_CKPT) return KDA_ERR_CHECKPOINT_CAPACITY;
    if (word & ERRBIT_BOUNDS) return KDA_ERR_DEBUG_BOUNDS;
    if (word & ERRBIT_ACCEPTED) return KDA_ERR_BAD_ACCEPTED;
    return KDA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// kda_fwd_noalloc: the tensor-core prefill with its scratch in a static array.
// ---------------------------------------------------------------------------
// In host code this name is only a host-side stand-in for the device array; its
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocMaxDevices = 64;

// The scratch array's device address is cached per device together with the
// unique id of the CUDA context it was looked up in (cuCtxGetId, reached through
// cudaGetDriverEntryPoint so the library needs no -lcuda).  A new context on the
// device -- after cudaDeviceReset, say -- has a new id and reloads the module, so
// the address is looked up again.  A failed lookup is not cached: the next call
// tries again.  Without the driver entry points the address is looked up on every
// call.
struct NoallocSlot {
    bool valid;
    unsigned long long ctx_id;
    void *ptr;
};
std::mutex g_noalloc_mu;
NoallocSlot g_noalloc_slot[kNoallocMaxDevices];

typedef int (*CtxGetCurrentFn)(void **);
typedef int (*CtxGetIdFn)(void *, unsigned long long *);

// Unique id of the current context; false when it cannot be read.
bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();   // a missing entry point is not an error of any later call
    });
    void *ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx) return false;
    return get_id(ctx, id) == 0;
}

// Device address of the static scratch in the current context (nullptr on error).
void *noalloc_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices)
        return nullptr;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocSlot &slot = g_noalloc_slot[dev];
    if (have_id && slot.valid && slot.ctx_id == id) return slot.ptr;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess) {
        cudaGetLastError();   // leave no error behind for a later launch check
        slot.valid = false;
        return nullptr;
    }
    slot.valid = have_id;
    slot.ctx_id = id;
    slot.ptr = p;
    return p;
}
}  // namespace

extern "C" kda_status kda_fwd_noalloc(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, const float *h0,
                                      const int32_t *cu_seqlens, int num_seqs, int B, int T,
                                      int H, int dk, int dv, int dtype, void *o, float *hT,
                                      void *stream) {
    // Host-side checks first, with a placeholder (aligned, non-null) workspace of
    // unbounded size, so bad arguments return before any CUDA call.
    int N;
    WsLayout L;
    void *placeholder = reinterpret_cast<void *>(uintptr_t(256));
    kda_status st = validate_fwd(q, k, v, g, beta, h0, cu_seqlens, num_seqs, B, T, H, dk, dv,
                                 dtype, o, hT, placeholder, SIZE_MAX, true, true, &N, &L,
                                 /*nseg_req=*/1);   // never T-split: scratch holds records only
    if (st != KDA_OK) return st;
    if (!is_tc_path(dtype, dk)) return KDA_ERR_UNSUPPORTED_SHAPE;
    if (L.total > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_EXCEEDS_STATIC_SCRATCH;
    if (N == 0) return KDA_OK;
    void *scratch = noalloc_scratch();
    if (!scratch) return KDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = tc_intra(q, k, v, g, beta, cu_seqlens, N, T, H, L, scratch, s)) != KDA_OK)
        return st;
    return tc_inter(h0, cu_seqlens, N, T, H, L, o, hT, scratch, s);
}
