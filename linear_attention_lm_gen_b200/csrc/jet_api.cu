// C ABI of the JetBlock token mixer: argument checks, kernel selection and
// launches. Declarations and the contract are in include/jet.h.
#include "jet.h"

#include <cuda.h>
#include <cublas_v2.h>
#include <dlfcn.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "common.cuh"
#include "k_decode.cuh"
#include "k_gen.cuh"
#include "k_genconv.cuh"
#include "k_genconv_decode.cuh"
#include "k_layer.cuh"
#include "k_prefill_simt.cuh"
#include "k_prefill_chain.cuh"
#include "k_prefill_correct.cuh"
#include "k_prefill_ws.cuh"
#include "k_segcombine.cuh"

using namespace jet;

namespace {

std::atomic<uint64_t> g_launches{0};

constexpr long long kMaxElems = (1LL << 62);

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool mul_ok(long long& acc, long long v) {
    if (v <= 0) return false;
    if (acc > kMaxElems / v) return false;
    acc *= v;
    return true;
}

// product of positive dimensions, or -1 on overflow / non-positive
long long elems(std::initializer_list<long long> dims) {
    long long acc = 1;
    for (long long d : dims)
        if (!mul_ok(acc, d)) return -1;
    return acc;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

size_t esize(jet_dtype dt) { return dt == JET_BF16 ? 2 : 4; }

jet_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? JET_OK : JET_ERR_CUDA;
}

// Launch with programmatic stream serialization allowed (the kernels wait
// for the previous kernel on the stream with pdl_wait before reading global
// memory), counting the launch.
template <typename... KArgs, typename... Args>
jet_status launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return JET_ERR_CUDA;
    return launch_status();
}

// opt a kernel into more than 48 KB of dynamic shared memory
template <typename K>
jet_status smem_attr(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return JET_OK;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) == cudaSuccess
               ? JET_OK : JET_ERR_CUDA;
}

bool dtype_ok(jet_dtype dt) { return dt == JET_F32 || dt == JET_BF16; }

// ---------------------------------------------------------------- K1
template <typename T, int TB, int RUN>
jet_status launch_genconv_t(const void* x, const void* w1, const void* w2, const void* v, const void* hin,
                            void* vout, void* hout, float* cw, int B, int Tn, int D, int H, int dv, int groups,
                            int hpc, cudaStream_t s, const int* slots, int n_slots) {
    const long long N = (long long)B * Tn;
    const size_t smem = sizeof(float) * gc_smem_floats(TB, hpc * GC_W);
    auto kern = genconv_kernel<T, TB, RUN>;
    if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
    // the head-group CTAs of a token block form one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + TB - 1) / TB), (unsigned)groups);
    cfg.blockDim = dim3(GC_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)groups;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, (const T*)x, (const T*)w1, (const T*)w2, (const T*)v,
                                             (const T*)hin, (T*)vout, (T*)hout, cw, B, Tn, D, H, dv, hpc, slots,
                                             n_slots);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return JET_ERR_CUDA;
    return launch_status();
}

// One new token per sequence, bf16: the decode kernel (one round trip to
// memory). Returns JET_ERR_UNSUPPORTED, before any launch, where its
// alignment or shared-memory needs are not met (the caller then takes the
// general kernel).
template <int TB>
jet_status launch_genconv_decode_t(const void* x, const void* w1, const void* w2, const void* v, const void* hin,
                                   void* vout, void* hout, float* cw, int B, int D, int H, int dv, int groups,
                                   int hpc, int per, size_t smem, cudaStream_t s, const int* slots, int n_slots) {
    auto kern = gcd::genconv_decode_kernel<TB>;
    if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((B + TB - 1) / TB), (unsigned)groups);
    cfg.blockDim = dim3(gcd::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)groups;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, (const __nv_bfloat16*)x, (const __nv_bfloat16*)w1,
                                             (const __nv_bfloat16*)w2, (const __nv_bfloat16*)v,
                                             (const __nv_bfloat16*)hin, (__nv_bfloat16*)vout, (__nv_bfloat16*)hout, cw,
                                             B, D, H, dv, hpc, per, slots, n_slots);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) return JET_ERR_CUDA;
    return launch_status();
}

jet_status launch_genconv_decode(const void* x, const void* w1, const void* w2, const void* v, const void* hin,
                                 void* vout, void* hout, float* cw, int B, int D, int H, int dv, cudaStream_t s,
                                 const int* slots, int n_slots) {
    if (!aligned_to(w1, 16) || !aligned_to(w2, 8) || (v && dv % 8 != 0)) return JET_ERR_UNSUPPORTED;
    const int TB = B <= 512 ? 8 : 16;
    const long long nblk = ((long long)B + TB - 1) / TB;
    // head groups (= cluster size, at most 8): enough CTAs to cover the SMs
    // about twice, then as few groups as give every group a head
    int groups = 1;
    while (groups < H && groups < 8 && nblk * groups < 296) ++groups;
    const int hpc = (H + groups - 1) / groups;
    groups = (H + hpc - 1) / hpc;
    const int per = (D / 16 + groups - 1) / groups;
    const size_t smem = gcd::layout(per * 16, hpc * GC_W).bytes;
    if (smem > 200 * 1024 || nblk > 0x7fffffffLL) return JET_ERR_UNSUPPORTED;
    return TB == 8 ? launch_genconv_decode_t<8>(x, w1, w2, v, hin, vout, hout, cw, B, D, H, dv, groups, hpc, per, smem,
                                                s, slots, n_slots)
                   : launch_genconv_decode_t<16>(x, w1, w2, v, hin, vout, hout, cw, B, D, H, dv, groups, hpc, per,
                                                 smem, s, slots, n_slots);
}

template <typename T>
jet_status launch_genconv(const void* x, const void* w1, const void* w2, const void* v, const void* hin,
                          void* vout, void* hout, float* cw, int B, int Tn, int D, int H, int dv,
                          cudaStream_t s, const int* slots = nullptr, int n_slots = 0) {
    if (std::is_same<T, __nv_bfloat16>::value && Tn == 1) {
        const jet_status st = launch_genconv_decode(x, w1, w2, v, hin, vout, hout, cw, B, D, H, dv, s, slots, n_slots);
        if (st != JET_ERR_UNSUPPORTED) return st;
    }
    constexpr int TB = 16;
    // a state-cache slot index applies to one token per sequence only (the
    // one-token work items look the slot up per item)
    if (slots && Tn != 1) return JET_ERR_UNSUPPORTED;
    const long long nblk = ((long long)B * Tn + TB - 1) / TB;
    // head groups (= cluster size, at most 8): enough CTAs to cover the SMs
    // about twice, then as few groups as give every group a head
    int groups = 1;
    while (groups < H && groups < 8 && nblk * groups < 296) ++groups;
    const int hpc = (H + groups - 1) / groups;
    groups = (H + hpc - 1) / hpc;
    if (Tn >= 8)   // (no slots here: checked above)
        return launch_genconv_t<T, TB, 8>(x, w1, w2, v, hin, vout, hout, cw, B, Tn, D, H, dv, groups, hpc, s,
                                          nullptr, 0);
    return launch_genconv_t<T, TB, 1>(x, w1, w2, v, hin, vout, hout, cw, B, Tn, D, H, dv, groups, hpc, s, slots,
                                      n_slots);
}

// prompts of at least this many tokens give every SM two 128-token generator CTAs
constexpr long long kGenWideTokens = 32768;
// the generator alone over a prompt (bf16): one CTA per 32 (or 128) tokens
jet_status launch_gen(const void* x, const void* w1, const void* w2, float* taps, int B, int Tn, int D, int H,
                      cudaStream_t s) {
    const long long N = (long long)B * Tn;
    const int HW4 = H * GC_W;
    if (N >= kGenWideTokens) {   // long prompts: 128-token CTAs, W1 read once per 128 tokens
        const size_t smem = kgen::wide_smem_bytes();
        if (smem_attr(kgen::gen_wide_kernel, smem) != JET_OK) return JET_ERR_CUDA;
        return launch(kgen::gen_wide_kernel, dim3((unsigned)((N + kgen::WGT - 1) / kgen::WGT)), dim3(kgen::THREADS),
                      smem, s, (const __nv_bfloat16*)x, (const __nv_bfloat16*)w1, (const __nv_bfloat16*)w2, taps, N,
                      D, HW4);
    }
    const size_t smem = kgen::smem_bytes(HW4);
    if (smem_attr(kgen::gen_kernel, smem) != JET_OK) return JET_ERR_CUDA;
    return launch(kgen::gen_kernel, dim3((unsigned)((N + kgen::GT - 1) / kgen::GT)), dim3(kgen::THREADS), smem, s,
                  (const __nv_bfloat16*)x, (const __nv_bfloat16*)w1, (const __nv_bfloat16*)w2, taps, N, D, HW4);
}
// prompts long enough to fill the GPU with 32-token CTAs take the stand-alone generator
constexpr long long kGenMinTokens = 1024;

jet_status check_gen(const void* x, const void* w1, const void* w2, int B, int T, int D, int H,
                     int hidden, int width, jet_dtype dt) {
    if (!x || !w1 || !w2) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, T, D}) < 0 || elems({B, T, H, 4}) < 0) return JET_ERR_INVALID_ARG;
    if (hidden != GC_HID || width != GC_W || D % 16 != 0 || H > 64) return JET_ERR_UNSUPPORTED;
    if ((long long)(B) * T / 16 + 1 > 0x7fffffffLL) return JET_ERR_UNSUPPORTED;
    const size_t es = dt == JET_BF16 ? 2 : 4;
    if (!aligned16(x) || !aligned_to(w1, es) || !aligned_to(w2, es)) return JET_ERR_MISALIGNED;
    return JET_OK;
}

// ---------------------------------------------------------------- K2
template <typename T, int DK>
jet_status launch_prefill_simt(const void* q, const void* k, const void* v, const float* g, const float* beta,
                               const float* S0, void* o, float* S_out, int B, int Tn, int H, int dv,
                               cudaStream_t s) {
    const size_t smem = sizeof(float) * ps_smem_floats(DK);
    auto kern = gdn_prefill_simt_kernel<T, DK>;
    if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
    return launch(kern, dim3(dv / PS_DVS, H, B), dim3(PS_THREADS), smem, s, (const T*)q, (const T*)k, (const T*)v, g,
                  beta, S0, (T*)o, S_out, Tn, H, dv);
}

// ---- TMA descriptors (driver entry point fetched once through the runtime)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return (EncodeTiledFn)p;
    }();
    return fn;
}

// bf16 tensor [rows][H][d] viewed as 3-D (d, H, rows); box (64, 1, box_rows), 128-byte swizzle
bool tile_map(CUtensorMap* m, const void* base, int d, int H, long long rows, int box_rows = 64) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * H * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Segment plans of the sequence-parallel prefill (P = 1: a single segment).
// Both keep every launch within one wave of the SMs and every segment at
// least 8 chunks long, and are functions of the shapes and the SM count only,
// so the workspace can be queried without a device: the queries plan for
// kMaxSMs (a full B200); a launch plans for min(the device's SMs, kMaxSMs),
// which never needs more workspace.
//   two passes (the fused low-memory kernel): phase A runs segments 0..P-2
//     with a transition slice each for p >= 1, phase C all P segments;
//   one pass (chunk images + chain kernel): all P segments at once, each with
//     a transition slice for p >= 1 (see k_prefill_chain.cuh).
constexpr int kMaxSMs = 148;
constexpr int kMinSegChunks = 8;
struct SegPlan { int P, seg_chunks; };
template <typename Fits>
SegPlan plan_segments(int T, Fits fits) {
    const int nch = (T + 63) / 64;
    SegPlan best{1, nch};
    for (int P = 2; P <= 64; ++P) {
        const int segc = (nch + P - 1) / P;
        if (segc < kMinSegChunks) break;
        const int Peff = (nch + segc - 1) / segc;
        if (Peff != P) continue;
        if (!fits(P)) break;
        best = SegPlan{P, segc};
    }
    return best;
}
SegPlan plan_two_pass(int B, int T, int H, int dv, int sms) {
    const int ns = dv / pfws::ROWS;
    return plan_segments(T, [&](int P) {
        return (long long)B * H * ((P - 1) * ns + (P - 2)) <= sms && (long long)B * H * ns * P <= sms;
    });
}
SegPlan plan_one_pass(int B, int T, int H, int dv, int sms) {
    const int ns = dv / pfws::ROWS;
    return plan_segments(T, [&](int P) { return (long long)B * H * ((long long)ns * P + P - 1) <= sms; });
}
// SMs a launch plans for (the current device's count, at most kMaxSMs)
int launch_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || n <= 0)
        return kMaxSMs;
    return std::min(n, kMaxSMs);
}
bool tc_prefill_ok(jet_dtype dt, int dk, int dv, long long BT) {
    return dt == JET_BF16 && dv % pfws::ROWS == 0 && (dk == 64 || dk == 96 || dk == 128) && BT < (1LL << 31);
}
// segment buffers of the two-pass plan: E [B][P-1][H][dv][dk] phase-A end
// states, A [B][P-1][H][dk][dk+8] transitions, S_start [B][P][H][dv][dk]
size_t seg_workspace_floats(int B, int H, int dk, int dv, int P) {
    if (P <= 1) return 0;
    return (size_t)B * (P - 1) * H * dv * dk      // E: phase A end states
         + (size_t)B * (P - 1) * H * dk * pfws::trans_ld(dk)   // A: transitions (padded rows)
         + (size_t)B * P * H * dv * dk;           // start states
}
// segment buffers of the one-pass plan, each part 1024-byte aligned:
// E [B][P][H][dv][dk], A [B][P][H][dk][dk+8] (float32), start states Sb
// [B][P][H][dv][dk] and Qe [B][H][nct][64][dk] (bf16)
struct OnePassLayout { size_t E, A, Sb, Qe, bytes; };
// nsegs: segments over all sequences, nchunks: chunks over all sequences
OnePassLayout one_pass_layout_n(size_t nsegs, size_t nchunks, int H, int dk, int dv) {
    auto up = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    OnePassLayout l{0, 0, 0, 0, 0};
    l.E = 0;
    l.A = l.E + up(sizeof(float) * nsegs * H * (size_t)dv * dk);
    l.Sb = l.A + up(sizeof(float) * nsegs * H * (size_t)dk * pfws::trans_ld(dk));
    l.Qe = l.Sb + up(sizeof(__nv_bfloat16) * nsegs * H * (size_t)dv * dk);
    l.bytes = l.Qe + up(sizeof(__nv_bfloat16) * nchunks * H * 64 * (size_t)dk);
    return l;
}
OnePassLayout one_pass_layout(int B, int T, int H, int dk, int dv, int P) {
    if (P <= 1) return OnePassLayout{0, 0, 0, 0, 0};
    return one_pass_layout_n((size_t)B * P, (size_t)B * ((T + 63) / 64), H, dk, dv);
}

// Segment plan of a variable-length batch (host cu_seqlens, already checked):
// one segment length for all sequences, the shortest (at least 8 chunks) that
// keeps the one-pass chain within one wave (value slices of every segment plus
// a transition slice for every segment after a sequence's first); if none
// does, one segment per sequence. Fills the chunk and segment offsets.
void plan_varlen(const int* cu, int nseq, int H, int dv, int sms, pfws::SeqMap& sq) {
    const int ns = dv / pfws::ROWS;
    int maxc = 1;
    sq.nseq = nseq;
    sq.chunk[0] = 0;
    for (int i = 0; i < nseq; ++i) {
        sq.tok[i] = cu[i];
        const int nci = (cu[i + 1] - cu[i] + 63) / 64;
        sq.chunk[i + 1] = sq.chunk[i] + nci;
        maxc = std::max(maxc, nci);
    }
    sq.tok[nseq] = cu[nseq];
    int segc = maxc;
    for (int cand = kMinSegChunks; cand < maxc; cand += std::max(1, cand / 2)) {
        long long ctas = 0;
        for (int i = 0; i < nseq; ++i) {
            const int Pi = (sq.chunk[i + 1] - sq.chunk[i] + cand - 1) / cand;
            ctas += (long long)H * ((long long)ns * Pi + Pi - 1);
        }
        if (ctas <= sms) { segc = cand; break; }
    }
    sq.seg_chunks = segc;
    sq.seg[0] = 0;
    for (int i = 0; i < nseq; ++i) sq.seg[i + 1] = sq.seg[i] + (sq.chunk[i + 1] - sq.chunk[i] + segc - 1) / segc;
}

// per-chunk image of the two-kernel plan (preparation + chain), bytes
size_t img_chunk_bytes(int dk) {
    switch (dk) {
        case 64: return pfws::Img<64>::BYTES;
        case 96: return pfws::Img<96>::BYTES;
        default: return pfws::Img<128>::BYTES;
    }
}
size_t split_img_bytes(int B, int T, int H, int dk) {
    return (size_t)B * H * ((T + pfws::C - 1) / pfws::C) * img_chunk_bytes(dk);
}

// Tensor-core prefill. SPLIT: K2a prepares every chunk into an image, then
// the chain kernel K2b runs every segment in one pass; with several segments
// the combine chains their start states and the correction kernel adds the
// start-state term to the outputs (workspace = images + one-pass buffers).
// Otherwise the fused kernel prepares chunk c+1 while it runs chunk c, in two
// passes over the segments (workspace = two-pass segment buffers only).
// CONV (split plan only): v is the raw V; the preparation folds the dynamic
// conv with `taps` into the chunk images and the chain reads the values
// before each segment (and the history of `cv`) for it.
// o += Qe S*^T for chunks chunk0 .. nct-1 (S* of chunk gc: entry gc / segc of
// Sb), or (variable length, vchunks > 0) for every chunk of the sequence map
template <int DK, int DV>
jet_status launch_correct(const __nv_bfloat16* Qe, const __nv_bfloat16* Sb, void* o, int B, int Tn, int H, int nct,
                          int chunk0, int segc, int P, cudaStream_t s, const pfws::SeqMap& sq, int vchunks) {
    if (vchunks == 0) {   // dense: groups of consecutive chunks of one segment per CTA
        auto kern = pfcor::prefill_correct_group_kernel<DK, DV>;
        const size_t smem = pfcor::smem_group_bytes(DK, DV);
        if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
        const int nseg = (nct + segc - 1) / segc - chunk0 / segc;
        // one wave: (segment, head, sequence) pairs times groups per segment within the SMs
        const long long pairs = (long long)nseg * H * B;
        const int gmax = (int)std::max<long long>(1, launch_sms() / std::max<long long>(1, pairs));
        const int ch = std::max(1, (segc + gmax - 1) / gmax);
        const int gps = (segc + ch - 1) / ch;
        return launch(kern, dim3(nseg * gps, H, B), dim3(pfcor::GTHREADS), smem, s, Qe, Sb, (__nv_bfloat16*)o, Tn, H,
                      nct, chunk0, segc, P, ch);
    }
    auto kern = pfcor::prefill_correct_kernel<DK, DV>;
    const size_t smem = pfcor::smem_bytes(DK, DV);
    if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
    const dim3 grid = vchunks > 0 ? dim3(vchunks, H, 1) : dim3(nct - chunk0, H, B);
    return launch(kern, grid, dim3(pfcor::THREADS), smem, s, Qe, Sb, (__nv_bfloat16*)o, Tn, H, nct, chunk0, segc, P,
                  sq);
}
template <int DK>
jet_status dispatch_correct(const __nv_bfloat16* Qe, const __nv_bfloat16* Sb, void* o, int B, int Tn, int H, int dv,
                            int nct, int chunk0, int segc, int P, cudaStream_t s, const pfws::SeqMap& sq,
                            int vchunks) {
    return dv == 256 ? launch_correct<DK, 256>(Qe, Sb, o, B, Tn, H, nct, chunk0, segc, P, s, sq, vchunks)
                     : launch_correct<DK, 128>(Qe, Sb, o, B, Tn, H, nct, chunk0, segc, P, s, sq, vchunks);
}
const pfws::SeqMap& no_seqmap() {   // nseq = 0: the dense layout
    static pfws::SeqMap m = [] {
        pfws::SeqMap z;
        memset(&z, 0, sizeof(z));
        return z;
    }();
    return m;
}

// range mode of the split plan: one segment, plus its transition A [B][H][dk][dk]
// and output corrections Qe [B][H][nct][64][dk] when A is given (S_out then
// receives the end state reached from S0, or from zero)
struct RangeOut {
    float* A;
    __nv_bfloat16* Qe;
    bool on;
};

template <int DK, bool SPLIT, bool CONV = false>
jet_status launch_prefill_tc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             const float* S0, void* o, float* S_out, void* workspace, int B, int Tn, int H,
                             int dv, cudaStream_t s, const float* taps = nullptr,
                             const pfch::ChainConv& cv = pfch::ChainConv{}, const RangeOut& range = RangeOut{},
                             const pfws::SeqMap* vsq = nullptr) {
    static_assert(SPLIT || !CONV, "the conv is folded in by the preparation kernel of the split plan");
    const pfws::SeqMap& sq = vsq ? *vsq : no_seqmap();
    CUtensorMap mq, mk, mv, mvh, mhh;
    const long long rows = vsq ? (long long)vsq->tok[vsq->nseq] : (long long)B * Tn;
    const int nseqs = vsq ? vsq->nseq : B;
    if (!tile_map(&mq, q, DK, H, rows) || !tile_map(&mk, k, DK, H, rows) || !tile_map(&mv, v, dv, H, rows))
        return JET_ERR_CUDA;
    // 16-row boxes of V and of the history (the values before a segment)
    mvh = mv;
    mhh = mv;
    if (CONV && (!tile_map(&mvh, v, dv, H, rows, 16) ||
                 (cv.hist_in && !tile_map(&mhh, cv.hist_in, dv, H, (long long)nseqs * 3, 16))))
        return JET_ERR_CUDA;
    if (CONV && !cv.hist_in) mhh = mvh;
    const int ns = dv / pfws::ROWS;
    const int nct = (Tn + pfws::C - 1) / pfws::C;
    const int sms = launch_sms();
    if (SPLIT) {
        auto chain = pfch::gdn_prefill_chain_kernel<DK, CONV>;
        constexpr uint32_t smem = pfch::ChainSmem<DK>::BYTES;
        if (smem_attr(chain, smem) != JET_OK) return JET_ERR_CUDA;
        const long long nchunks = vsq ? vsq->chunk[vsq->nseq] : (long long)B * nct;   // over all sequences
        uint8_t* img = static_cast<uint8_t*>(workspace);
        uint8_t* segws = img + (size_t)nchunks * H * img_chunk_bytes(DK);
        {   // K2a: every chunk of every (sequence, head)
            auto prep = pfws::gdn_chunk_prep_kernel<DK>;
            if (smem_attr(prep, pfws::PrepSmem<DK>::BYTES) != JET_OK) return JET_ERR_CUDA;
            const long long items = nchunks * H;
            const int grid = (int)std::min<long long>(items, (long long)pfws::PREP_CTAS * sms);   // resident CTAs
            if (launch(prep, dim3(grid), dim3(pfws::PREP_THREADS), pfws::PrepSmem<DK>::BYTES, s, mq, mk, g, beta,
                       CONV ? taps : nullptr, (int)(cv.hist_in != nullptr), img, Tn, H, nct, (int)items,
                       sq, (int)CONV) != JET_OK)
                return JET_ERR_CUDA;
        }
        if (vsq) {   // variable length: the segments of the plan in the sequence map
            const int nsegs = vsq->seg[vsq->nseq];
            const bool multi = nsegs > vsq->nseq;
            const OnePassLayout lay = one_pass_layout_n(nsegs, nchunks, H, DK, dv);
            float* E = reinterpret_cast<float*>(segws + lay.E);
            float* A = reinterpret_cast<float*>(segws + lay.A);
            __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(segws + lay.Sb);
            __nv_bfloat16* Qe = reinterpret_cast<__nv_bfloat16*>(segws + lay.Qe);
            const pfch::ChainSeg seg{1, vsq->seg_chunks, E, A, Qe, pfws::trans_ld(DK), 0};
            if (launch(chain, dim3(ns + (multi ? 1 : 0), H, nsegs), dim3(pfch::THREADS), smem, s, mk, mv, mvh, mhh,
                       (const uint8_t*)img, S0, (__nv_bfloat16*)o, S_out, Tn, H, dv, seg, cv, sq) != JET_OK)
                return JET_ERR_CUDA;
            if (!multi) return JET_OK;
            const size_t sc_smem = sc_smem_bytes(DK);
            if (smem_attr(seg_combine_kernel<DK, true>, sc_smem) != JET_OK) return JET_ERR_CUDA;
            if (launch(seg_combine_kernel<DK, true>, dim3(dv / SC_ROWS, H, vsq->nseq), dim3(sc_threads(DK)), sc_smem,
                       s, (const float*)E, (const float*)A, (const float*)nullptr, (float*)nullptr, Sb, S_out, 0, H,
                       dv, CombineLayout{0, pfws::trans_ld(DK)}, sq) != JET_OK)
                return JET_ERR_CUDA;
            return dispatch_correct<DK>(Qe, Sb, o, 1, Tn, H, dv, (int)nchunks, 0, vsq->seg_chunks, 1, s, sq,
                                        (int)nchunks);
        }
        if (range.on) {   // one segment; the transition slice when A is wanted
            const bool tr = range.A != nullptr;
            const pfch::ChainSeg seg{1, nct, nullptr, range.A, range.Qe, DK, tr ? 1 : 0};
            return launch(chain, dim3(ns + (tr ? 1 : 0), H, B), dim3(pfch::THREADS), smem, s, mk, mv, mvh, mhh,
                          (const uint8_t*)img, S0, (__nv_bfloat16*)o, S_out, Tn, H, dv, seg, cv, sq);
        }
        const SegPlan plan = plan_one_pass(B, Tn, H, dv, sms);
        const int P = plan.P;
        const OnePassLayout lay = one_pass_layout(B, Tn, H, DK, dv, P);
        float* E = reinterpret_cast<float*>(segws + lay.E);
        float* A = reinterpret_cast<float*>(segws + lay.A);
        __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(segws + lay.Sb);
        __nv_bfloat16* Qe = reinterpret_cast<__nv_bfloat16*>(segws + lay.Qe);
        const pfch::ChainSeg seg = P == 1 ? pfch::ChainSeg{1, plan.seg_chunks, nullptr, nullptr, nullptr, 0, 0}
                                          : pfch::ChainSeg{P, plan.seg_chunks, E, A, Qe, pfws::trans_ld(DK), 0};
        if (launch(chain, dim3(ns + (P > 1 ? 1 : 0), H, B * P), dim3(pfch::THREADS), smem, s, mk, mv, mvh, mhh,
                   (const uint8_t*)img, S0, (__nv_bfloat16*)o, S_out, Tn, H, dv, seg, cv, sq) != JET_OK)
            return JET_ERR_CUDA;
        if (P == 1) return JET_OK;
        // start states S*_1 .. S*_{P-1} and the final state
        const size_t sc_smem = sc_smem_bytes(DK);
        if (smem_attr(seg_combine_kernel<DK, true>, sc_smem) != JET_OK) return JET_ERR_CUDA;
        if (launch(seg_combine_kernel<DK, true>, dim3(dv / SC_ROWS, H, B), dim3(sc_threads(DK)), sc_smem, s,
                   (const float*)E, (const float*)A, (const float*)nullptr, (float*)nullptr, Sb, S_out, P, H, dv,
                   CombineLayout{0, pfws::trans_ld(DK)}, sq) != JET_OK)
            return JET_ERR_CUDA;
        // outputs of the segments p >= 1: O += Qe S*^T
        return dispatch_correct<DK>(Qe, Sb, o, B, Tn, H, dv, nct, plan.seg_chunks, plan.seg_chunks, P, s, sq, 0);
    }
    auto fused = pfws::gdn_prefill_ws_kernel<DK>;
    if (smem_attr(fused, pfws::SMEM_BYTES) != JET_OK) return JET_ERR_CUDA;
    float* ws = reinterpret_cast<float*>(workspace);
    auto run = [&](dim3 grid, const pfws::Seg& seg) {
        return launch(fused, grid, dim3(pfws::THREADS), pfws::SMEM_BYTES, s, mq, mk, mv, g, beta, S0,
                      (__nv_bfloat16*)o, S_out, Tn, H, dv, seg);
    };
    const SegPlan plan = plan_two_pass(B, Tn, H, dv, sms);
    const int P = plan.P;
    if (P == 1) return run(dim3(ns, H, B), pfws::Seg{1, plan.seg_chunks, 1, 0, nullptr, nullptr, nullptr});
    float* E = ws;
    float* A = E + (size_t)B * (P - 1) * H * dv * DK;
    float* Sst = A + (size_t)B * (P - 1) * H * DK * pfws::trans_ld(DK);
    // phase A: segments 0 .. P-2, value slices plus the transition slice
    if (run(dim3(ns + 1, H, B * (P - 1)), pfws::Seg{P, plan.seg_chunks, P - 1, 1, nullptr, E, A}) != JET_OK)
        return JET_ERR_CUDA;
    // start states of every segment (S0 copied for segment 0)
    const size_t sc_smem = sc_smem_bytes(DK);
    if (smem_attr(seg_combine_kernel<DK, false>, sc_smem) != JET_OK) return JET_ERR_CUDA;
    if (launch(seg_combine_kernel<DK, false>, dim3(dv / SC_ROWS, H, B), dim3(sc_threads(DK)), sc_smem, s,
               (const float*)E, (const float*)A, S0, Sst, (__nv_bfloat16*)nullptr, (float*)nullptr, P, H, dv,
               CombineLayout{0, pfws::trans_ld(DK)}, sq) != JET_OK)
        return JET_ERR_CUDA;
    // phase C: every segment from its start state, with outputs
    return run(dim3(ns, H, B * P), pfws::Seg{P, plan.seg_chunks, P, 0, Sst, nullptr, nullptr});
}

template <typename T>
jet_status dispatch_prefill(int dk, const void* q, const void* k, const void* v, const float* g,
                            const float* beta, const float* S0, void* o, float* S_out, int B, int Tn,
                            int H, int dv, cudaStream_t s) {
    switch (dk) {
#define JET_CASE(DK) case DK: return launch_prefill_simt<T, DK>(q, k, v, g, beta, S0, o, S_out, B, Tn, H, dv, s);
        JET_CASE(16) JET_CASE(32) JET_CASE(48) JET_CASE(64)
        JET_CASE(80) JET_CASE(96) JET_CASE(112) JET_CASE(128)
#undef JET_CASE
        default: return JET_ERR_UNSUPPORTED;
    }
}

// ---------------------------------------------------------------- K3
template <typename T, int NV>
jet_status launch_decode(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float* S, void* o, int B, int H, int dv, const DecConv* conv, cudaStream_t s,
                         const int* slots, int n_slots, int early) {
    const dim3 grid((dv + DEC_ROWS - 1) / DEC_ROWS, H, B);
    // the state stream wants the largest L1 (it holds the loads in flight): ask for the
    // smallest shared-memory carve-out, also while the previous launch's CTAs with a
    // large one still share the SM
    auto kern = conv ? gdn_decode_kernel<T, NV, true> : gdn_decode_kernel<T, NV>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 0) != cudaSuccess)
        return JET_ERR_CUDA;
    if (conv)
        return launch(gdn_decode_kernel<T, NV, true>, grid, dim3(DEC_THREADS), 0, s, (const T*)q, (const T*)k,
                      (const T*)v, g, beta, S, (T*)o, H, dv, *conv, slots, n_slots, early);
    return launch(gdn_decode_kernel<T, NV>, grid, dim3(DEC_THREADS), 0, s, (const T*)q, (const T*)k, (const T*)v, g,
                  beta, S, (T*)o, H, dv, DecConv{}, slots, n_slots, early);
}

template <typename T>
jet_status dispatch_decode(int dk, const void* q, const void* k, const void* v, const float* g,
                           const float* beta, float* S, void* o, int B, int H, int dv, cudaStream_t s,
                           const DecConv* conv = nullptr, const int* slots = nullptr, int n_slots = 0,
                           int early = 0) {
    switch (dk / 16) {
#define JET_CASE(NV) case NV: return launch_decode<T, NV>(q, k, v, g, beta, S, o, B, H, dv, conv, s, slots, n_slots, early);
        JET_CASE(1) JET_CASE(2) JET_CASE(3) JET_CASE(4) JET_CASE(5) JET_CASE(6) JET_CASE(7) JET_CASE(8)
#undef JET_CASE
        default: return JET_ERR_UNSUPPORTED;
    }
}

bool shape_ok(int dk, int dv) { return dk % 16 == 0 && dk >= 16 && dk <= 128 && dv % 32 == 0 && dv <= 256; }

}  // namespace

extern "C" {

jet_status jet_kernel_gen(const void* x, const void* w1, const void* w2, float* conv_w, int B, int T, int D,
                          int H, int hidden, int width, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, T, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!conv_w) return JET_ERR_INVALID_ARG;
    if (!aligned_to(conv_w, 4)) return JET_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == JET_BF16 && (long long)B * T >= kGenMinTokens) return launch_gen(x, w1, w2, conv_w, B, T, D, H, s);
    if (dt == JET_BF16)
        return launch_genconv<__nv_bfloat16>(x, w1, w2, nullptr, nullptr, nullptr, nullptr, conv_w, B, T, D, H, 32, s);
    return launch_genconv<float>(x, w1, w2, nullptr, nullptr, nullptr, nullptr, conv_w, B, T, D, H, 32, s);
}

jet_status jet_dyn_conv_v(const void* x, const void* w1, const void* w2, const void* v, const void* hist_in,
                          void* v_out, void* hist_out, float* conv_w_out, int B, int T, int D, int H, int dv,
                          int hidden, int width, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, T, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!v || !v_out) return JET_ERR_INVALID_ARG;
    const long long nv = elems({B, T, H, dv});
    const long long nh = elems({B, 3, H, dv});
    if (nv < 0 || nh < 0) return JET_ERR_INVALID_ARG;
    if (dv % 32 != 0 || dv > 256) return JET_ERR_UNSUPPORTED;
    for (const void* p : {v, (const void*)v_out, hist_in, (const void*)hist_out})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (conv_w_out && !aligned_to(conv_w_out, 4)) return JET_ERR_MISALIGNED;
    const size_t es = esize(dt);
    if (overlap(v, nv * es, v_out, nv * es)) return JET_ERR_INVALID_ARG;
    if (hist_in && hist_out && overlap(hist_in, nh * es, hist_out, nh * es)) return JET_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == JET_BF16)
        return launch_genconv<__nv_bfloat16>(x, w1, w2, v, hist_in, v_out, hist_out, conv_w_out, B, T, D, H, dv, s);
    return launch_genconv<float>(x, w1, w2, v, hist_in, v_out, hist_out, conv_w_out, B, T, D, H, dv, s);
}

size_t jet_gdn_prefill_workspace_min(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt) {
    if (B <= 0 || T <= 0 || H <= 0 || chunk != 64 || !tc_prefill_ok(dt, dk, dv, (long long)B * T)) return 0;
    const SegPlan plan = plan_two_pass(B, T, H, dv, kMaxSMs);
    return sizeof(float) * seg_workspace_floats(B, H, dk, dv, plan.P);
}

size_t jet_gdn_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt) {
    if (B <= 0 || T <= 0 || H <= 0 || chunk != 64 || !tc_prefill_ok(dt, dk, dv, (long long)B * T)) return 0;
    const SegPlan plan = plan_one_pass(B, T, H, dv, kMaxSMs);
    return split_img_bytes(B, T, H, dk) + one_pass_layout(B, T, H, dk, dv, plan.P).bytes;
}

jet_status jet_gdn_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                           const float* S0, void* o, float* S_out, void* workspace, size_t ws_bytes, int B,
                           int T, int H, int dk, int dv, int chunk, jet_dtype dt, void* stream) {
    if (!q || !k || !v || !g || !beta || !o || !S_out) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, T, H, dk}) < 0 || elems({B, T, H, dv}) < 0 || elems({B, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || chunk != 64 || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    for (const void* p : {q, k, v, (const void*)S0, (const void*)o, (const void*)S_out, (const void*)workspace})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4)) return JET_ERR_MISALIGNED;
    if (!workspace) ws_bytes = 0;
    const size_t need_min = jet_gdn_prefill_workspace_min(B, T, H, dk, dv, chunk, dt);
    if (ws_bytes < need_min) return JET_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tc_prefill_ok(dt, dk, dv, (long long)B * T)) {
        // tensor-core path: two-kernel plan when the workspace holds the chunk images
        const bool split = ws_bytes >= jet_gdn_prefill_workspace_size(B, T, H, dk, dv, chunk, dt);
#define JET_TC(DK)                                                                                     \
        return split ? launch_prefill_tc<DK, true>(q, k, v, g, beta, S0, o, S_out, workspace, B, T, H, dv, s) \
                     : launch_prefill_tc<DK, false>(q, k, v, g, beta, S0, o, S_out, workspace, B, T, H, dv, s);
        if (dk == 64) { JET_TC(64) }
        if (dk == 96) { JET_TC(96) }
        JET_TC(128)
#undef JET_TC
    }
    if (dt == JET_BF16)
        return dispatch_prefill<__nv_bfloat16>(dk, q, k, v, g, beta, S0, o, S_out, B, T, H, dv, s);
    return dispatch_prefill<float>(dk, q, k, v, g, beta, S0, o, S_out, B, T, H, dv, s);
}

// ---- generator + conv + GDN prefill in one call
// workspace: [taps B*T*H*4 float32 | rest], each part 1024-byte aligned; rest =
// the split-plan workspace of the tensor-core path (the chain applies the
// conv), else a v' buffer for the separate conv pass and the SIMT prefill
size_t jet_jetblock_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt) {
    if (B <= 0 || T <= 0 || H <= 0 || dv <= 0 || chunk != 64 || !dtype_ok(dt)) return 0;
    const long long nt = elems({B, T, H, 4}), nv = elems({B, T, H, dv});
    if (nt < 0 || nv < 0) return 0;
    auto up = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    const size_t taps = up((size_t)nt * sizeof(float));
    if (tc_prefill_ok(dt, dk, dv, (long long)B * T))
        return taps + jet_gdn_prefill_workspace_size(B, T, H, dk, dv, chunk, dt);
    return taps + up((size_t)nv * esize(dt));
}

jet_status jet_jetblock_prefill(const void* x, const void* w1, const void* w2, const void* q, const void* k,
                                const void* v, const void* hist_in, void* hist_out, const float* g,
                                const float* beta, const float* S0, void* o, float* S_out, void* workspace,
                                size_t ws_bytes, int B, int T, int D, int H, int dk, int dv, int hidden, int width,
                                int chunk, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, T, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!q || !k || !v || !g || !beta || !o || !S_out) return JET_ERR_INVALID_ARG;
    const long long nv = elems({B, T, H, dv}), nh = elems({B, 3, H, dv});
    if (elems({B, T, H, dk}) < 0 || nv < 0 || nh < 0 || elems({B, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || chunk != 64 || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    for (const void* p : {q, k, v, hist_in, (const void*)hist_out, (const void*)S0, (const void*)o,
                          (const void*)S_out, (const void*)workspace})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4)) return JET_ERR_MISALIGNED;
    const size_t es = esize(dt), vb = (size_t)nv * es, hb = (size_t)nh * es;
    // v is read (raw, and around segment starts) while o and the new history are written
    if (overlap(v, vb, o, vb)) return JET_ERR_INVALID_ARG;
    if (hist_out && (overlap(v, vb, hist_out, hb) || (hist_in && overlap(hist_in, hb, hist_out, hb))))
        return JET_ERR_INVALID_ARG;
    if (!workspace) ws_bytes = 0;
    if (ws_bytes < jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, chunk, dt)) return JET_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* taps = static_cast<float*>(workspace);
    uint8_t* rest = static_cast<uint8_t*>(workspace) + ((elems({B, T, H, 4}) * sizeof(float) + 1023) & ~size_t(1023));
    if (tc_prefill_ok(dt, dk, dv, (long long)B * T)) {
        st = (long long)B * T >= kGenMinTokens
                 ? launch_gen(x, w1, w2, taps, B, T, D, H, s)
                 : launch_genconv<__nv_bfloat16>(x, w1, w2, nullptr, nullptr, nullptr, nullptr, taps, B, T, D, H, dv, s);
        if (st != JET_OK) return st;
        const pfch::ChainConv cv{static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(hist_in),
                                 static_cast<__nv_bfloat16*>(hist_out)};
#define JET_TC(DK) \
        return launch_prefill_tc<DK, true, true>(q, k, v, g, beta, S0, o, S_out, rest, B, T, H, dv, s, taps, cv);
        if (dk == 64) { JET_TC(64) }
        if (dk == 96) { JET_TC(96) }
        JET_TC(128)
#undef JET_TC
    }
    // other shapes and float32: the conv pass writes v' into the workspace, then the SIMT prefill
    st = dt == JET_BF16
             ? launch_genconv<__nv_bfloat16>(x, w1, w2, v, hist_in, rest, hist_out, taps, B, T, D, H, dv, s)
             : launch_genconv<float>(x, w1, w2, v, hist_in, rest, hist_out, taps, B, T, D, H, dv, s);
    if (st != JET_OK) return st;
    if (dt == JET_BF16)
        return dispatch_prefill<__nv_bfloat16>(dk, q, k, rest, g, beta, S0, o, S_out, B, T, H, dv, s);
    return dispatch_prefill<float>(dk, q, k, rest, g, beta, S0, o, S_out, B, T, H, dv, s);
}

// ---- variable-length batch: sequences of different lengths packed along the token axis
namespace {
// host cu_seqlens: nseq + 1 offsets, 0 first, strictly increasing; the total token count
bool varlen_ok(const int* cu, int nseq, long long* total) {
    if (!cu || nseq < 1 || nseq > pfws::kMaxVarlenSeqs || cu[0] != 0) return false;
    for (int i = 0; i < nseq; ++i)
        if (cu[i + 1] <= cu[i]) return false;
    *total = cu[nseq];
    return *total > 0 && *total < (1LL << 31);
}
size_t varlen_workspace(const int* cu, int nseq, int H, int dk, int dv, int sms) {
    pfws::SeqMap sq;
    plan_varlen(cu, nseq, H, dv, sms, sq);
    const long long total = cu[nseq];
    auto up = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    const size_t nchunks = (size_t)sq.chunk[nseq];
    const size_t nsegs = (size_t)sq.seg[nseq];
    return up((size_t)total * H * 4 * sizeof(float)) + nchunks * H * img_chunk_bytes(dk) +
           (nsegs > (size_t)nseq ? one_pass_layout_n(nsegs, nchunks, H, dk, dv).bytes : 0);
}
}  // namespace

size_t jet_jetblock_prefill_varlen_workspace_size(const int* cu_seqlens, int nseq, int H, int dk, int dv, int chunk,
                                                  jet_dtype dt) {
    long long total = 0;
    if (H <= 0 || chunk != 64 || !varlen_ok(cu_seqlens, nseq, &total) || !tc_prefill_ok(dt, dk, dv, total)) return 0;
    return varlen_workspace(cu_seqlens, nseq, H, dk, dv, kMaxSMs);
}

jet_status jet_jetblock_prefill_varlen(const void* x, const void* w1, const void* w2, const void* q, const void* k,
                                       const void* v, const void* hist_in, void* hist_out, const float* g,
                                       const float* beta, const float* S0, void* o, float* S_out, void* workspace,
                                       size_t ws_bytes, const int* cu_seqlens, int nseq, int D, int H, int dk, int dv,
                                       int hidden, int width, int chunk, jet_dtype dt, void* stream) {
    long long total = 0;
    if (!cu_seqlens || nseq < 1) return JET_ERR_INVALID_ARG;
    if (nseq > pfws::kMaxVarlenSeqs) return JET_ERR_UNSUPPORTED;
    if (!varlen_ok(cu_seqlens, nseq, &total)) return JET_ERR_INVALID_ARG;
    jet_status st = check_gen(x, w1, w2, 1, (int)total, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!q || !k || !v || !g || !beta || !o || !S_out) return JET_ERR_INVALID_ARG;
    const long long nv = elems({total, H, dv}), nh = elems({nseq, 3, H, dv});
    if (elems({total, H, dk}) < 0 || nv < 0 || nh < 0 || elems({nseq, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || chunk != 64 || H > 65535) return JET_ERR_UNSUPPORTED;
    if (!tc_prefill_ok(dt, dk, dv, total)) return JET_ERR_UNSUPPORTED;
    for (const void* p : {q, k, v, hist_in, (const void*)hist_out, (const void*)S0, (const void*)o,
                          (const void*)S_out, (const void*)workspace})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4)) return JET_ERR_MISALIGNED;
    const size_t es = esize(dt), vb = (size_t)nv * es, hb = (size_t)nh * es;
    if (overlap(v, vb, o, vb)) return JET_ERR_INVALID_ARG;
    if (hist_out && (overlap(v, vb, hist_out, hb) || (hist_in && overlap(hist_in, hb, hist_out, hb))))
        return JET_ERR_INVALID_ARG;
    if (!workspace) ws_bytes = 0;
    if (ws_bytes < varlen_workspace(cu_seqlens, nseq, H, dk, dv, kMaxSMs)) return JET_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    pfws::SeqMap sq;
    plan_varlen(cu_seqlens, nseq, H, dv, launch_sms(), sq);
    float* taps = static_cast<float*>(workspace);
    uint8_t* rest = static_cast<uint8_t*>(workspace) + (((size_t)total * H * 4 * sizeof(float) + 1023) & ~size_t(1023));
    st = total >= kGenMinTokens
             ? launch_gen(x, w1, w2, taps, 1, (int)total, D, H, s)
             : launch_genconv<__nv_bfloat16>(x, w1, w2, nullptr, nullptr, nullptr, nullptr, taps, 1, (int)total, D, H,
                                             dv, s);
    if (st != JET_OK) return st;
    const pfch::ChainConv cv{static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(hist_in),
                             static_cast<__nv_bfloat16*>(hist_out)};
#define JET_TC(DK)                                                                                          \
    return launch_prefill_tc<DK, true, true>(q, k, v, g, beta, S0, o, S_out, rest, nseq, 0, H, dv, s, taps, cv, \
                                             RangeOut{}, &sq);
    if (dk == 64) { JET_TC(64) }
    if (dk == 96) { JET_TC(96) }
    JET_TC(128)
#undef JET_TC
}

// ---- sequence parallelism over token ranges (one range per GPU)
size_t jet_jetblock_prefill_range_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt) {
    if (B <= 0 || T <= 0 || H <= 0 || chunk != 64 || !tc_prefill_ok(dt, dk, dv, (long long)B * T)) return 0;
    const long long nt = elems({B, T, H, 4});
    if (nt < 0) return 0;
    return (((size_t)nt * sizeof(float) + 1023) & ~size_t(1023)) + split_img_bytes(B, T, H, dk);
}

jet_status jet_jetblock_prefill_range(const void* x, const void* w1, const void* w2, const void* q, const void* k,
                                      const void* v, const void* hist_in, void* hist_out, const float* g,
                                      const float* beta, const float* S0, void* o, float* E_out, float* A_out,
                                      void* Qe_out, void* workspace, size_t ws_bytes, int B, int T, int D, int H,
                                      int dk, int dv, int hidden, int width, int chunk, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, T, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!q || !k || !v || !g || !beta || !o || !E_out) return JET_ERR_INVALID_ARG;
    if ((A_out == nullptr) != (Qe_out == nullptr)) return JET_ERR_INVALID_ARG;
    const long long nv = elems({B, T, H, dv}), nh = elems({B, 3, H, dv});
    if (elems({B, T, H, dk}) < 0 || nv < 0 || nh < 0 || elems({B, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || chunk != 64 || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    if (!tc_prefill_ok(dt, dk, dv, (long long)B * T)) return JET_ERR_UNSUPPORTED;
    for (const void* p : {q, k, v, hist_in, (const void*)hist_out, (const void*)S0, (const void*)o,
                          (const void*)E_out, (const void*)A_out, (const void*)Qe_out, (const void*)workspace})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4)) return JET_ERR_MISALIGNED;
    const size_t es = esize(dt), vb = (size_t)nv * es, hb = (size_t)nh * es;
    if (overlap(v, vb, o, vb)) return JET_ERR_INVALID_ARG;
    if (hist_out && (overlap(v, vb, hist_out, hb) || (hist_in && overlap(hist_in, hb, hist_out, hb))))
        return JET_ERR_INVALID_ARG;
    if (!workspace) ws_bytes = 0;
    if (ws_bytes < jet_jetblock_prefill_range_workspace_size(B, T, H, dk, dv, chunk, dt)) return JET_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* taps = static_cast<float*>(workspace);
    uint8_t* rest = static_cast<uint8_t*>(workspace) + ((elems({B, T, H, 4}) * sizeof(float) + 1023) & ~size_t(1023));
    st = (long long)B * T >= kGenMinTokens
             ? launch_gen(x, w1, w2, taps, B, T, D, H, s)
             : launch_genconv<__nv_bfloat16>(x, w1, w2, nullptr, nullptr, nullptr, nullptr, taps, B, T, D, H, dv, s);
    if (st != JET_OK) return st;
    const pfch::ChainConv cv{static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(hist_in),
                             static_cast<__nv_bfloat16*>(hist_out)};
    const RangeOut range{A_out, static_cast<__nv_bfloat16*>(Qe_out), true};
#define JET_TC(DK) \
    return launch_prefill_tc<DK, true, true>(q, k, v, g, beta, S0, o, E_out, rest, B, T, H, dv, s, taps, cv, range);
    if (dk == 64) { JET_TC(64) }
    if (dk == 96) { JET_TC(96) }
    JET_TC(128)
#undef JET_TC
}

jet_status jet_gdn_range_compose(const float* E, const float* A, void* Sb_out, float* S_out, int R, int B, int H,
                                 int dk, int dv, void* stream) {
    if (!E || !A || !Sb_out || !S_out) return JET_ERR_INVALID_ARG;
    if (R < 2 || elems({R, B, H, dv, dk}) < 0 || elems({R, B, H, dk, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!(dk == 64 || dk == 96 || dk == 128) || dv % SC_ROWS != 0 || dv > 256 || B > 65535 || H > 65535)
        return JET_ERR_UNSUPPORTED;
    for (const void* p : {(const void*)E, (const void*)A, (const void*)Sb_out, (const void*)S_out})
        if (!aligned16(p)) return JET_ERR_MISALIGNED;
    const size_t sb = (size_t)R * B * H * dv * dk;
    if (overlap(E, sb * 4, S_out, (size_t)B * H * dv * dk * 4) || overlap(E, sb * 4, Sb_out, sb * 2))
        return JET_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto run = [&](auto kern, int DK) {
        const size_t smem = sc_smem_bytes(DK);
        if (smem_attr(kern, smem) != JET_OK) return JET_ERR_CUDA;
        return launch(kern, dim3(dv / SC_ROWS, H, B), dim3(sc_threads(DK)), smem, s, E, A, (const float*)nullptr,
                      (float*)nullptr, static_cast<__nv_bfloat16*>(Sb_out), S_out, R, H, dv, CombineLayout{1, DK},
                      no_seqmap());
    };
    if (dk == 64) return run(seg_combine_kernel<64, true>, 64);
    if (dk == 96) return run(seg_combine_kernel<96, true>, 96);
    return run(seg_combine_kernel<128, true>, 128);
}

jet_status jet_gdn_range_correct(const void* Qe, const void* Sb, void* o, int B, int T, int H, int dk, int dv,
                                 jet_dtype dt, void* stream) {
    if (!Qe || !Sb || !o) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, T, H, dv}) < 0 || elems({B, H, dv, dk}) < 0 || elems({B, H, T, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!tc_prefill_ok(dt, dk, dv, (long long)B * T) || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    for (const void* p : {Qe, Sb, (const void*)o})
        if (!aligned16(p)) return JET_ERR_MISALIGNED;
    const size_t ob = (size_t)B * T * H * dv * 2;
    if (overlap(o, ob, Qe, (size_t)B * H * ((T + 63) / 64) * 64 * dk * 2) || overlap(o, ob, Sb, (size_t)B * H * dv * dk * 2))
        return JET_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nct = (T + 63) / 64;
    const __nv_bfloat16* qe = static_cast<const __nv_bfloat16*>(Qe);
    const __nv_bfloat16* sb = static_cast<const __nv_bfloat16*>(Sb);
    if (dk == 64) return dispatch_correct<64>(qe, sb, o, B, T, H, dv, nct, 0, nct, 1, s, no_seqmap(), 0);
    if (dk == 96) return dispatch_correct<96>(qe, sb, o, B, T, H, dv, nct, 0, nct, 1, s, no_seqmap(), 0);
    return dispatch_correct<128>(qe, sb, o, B, T, H, dv, nct, 0, nct, 1, s, no_seqmap(), 0);
}

jet_status jet_gdn_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                               float* S, void* o, int B, int H, int dk, int dv, jet_dtype dt, void* stream) {
    if (!q || !k || !v || !g || !beta || !S || !o) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    const size_t es = esize(dt);
    for (const void* p : {q, k, v, (const void*)o})
        if (!aligned_to(p, es)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4) || !aligned16(S)) return JET_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == JET_BF16) return dispatch_decode<__nv_bfloat16>(dk, q, k, v, g, beta, S, o, B, H, dv, s);
    return dispatch_decode<float>(dk, q, k, v, g, beta, S, o, B, H, dv, s);
}

jet_status jet_conv_gdn_decode_step(const void* q, const void* k, const void* v, const void* hist_in,
                                    void* hist_out, const float* taps, const float* g, const float* beta, float* S,
                                    void* o, int B, int H, int dk, int dv, jet_dtype dt, void* stream) {
    if (!q || !k || !v || !g || !beta || !S || !o || !hist_out || !taps) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, H, dv, dk}) < 0 || elems({B, 3, H, dv}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    const size_t es = esize(dt);
    for (const void* p : {q, k, v, hist_in, (const void*)hist_out, (const void*)o})
        if (p && !aligned_to(p, es)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4) || !aligned16(S) || !aligned16(taps)) return JET_ERR_MISALIGNED;
    const size_t nh = (size_t)B * 3 * H * dv * es;
    if (hist_in && overlap(hist_in, nh, hist_out, nh)) return JET_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const DecConv conv{taps, hist_in, hist_out};
    if (dt == JET_BF16) return dispatch_decode<__nv_bfloat16>(dk, q, k, v, g, beta, S, o, B, H, dv, s, &conv);
    return dispatch_decode<float>(dk, q, k, v, g, beta, S, o, B, H, dv, s, &conv);
}

jet_status jet_jetblock_decode_step(const void* x, const void* w1, const void* w2, const void* q, const void* k,
                                    const void* v, const void* hist_in, void* hist_out, const float* g,
                                    const float* beta, float* S, void* o, float* taps, int B, int D, int H, int dk,
                                    int dv, int hidden, int width, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, 1, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!taps) return JET_ERR_INVALID_ARG;
    if (!aligned16(taps)) return JET_ERR_MISALIGNED;
    // validate the decode half before launching anything (no sizes / buffers change between the two)
    if (!q || !k || !v || !g || !beta || !S || !o || !hist_out) return JET_ERR_INVALID_ARG;
    if (elems({B, H, dv, dk}) < 0 || elems({B, 3, H, dv}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    const size_t es = esize(dt);
    for (const void* p : {q, k, v, hist_in, (const void*)hist_out, (const void*)o})
        if (p && !aligned_to(p, es)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4) || !aligned16(S)) return JET_ERR_MISALIGNED;
    const size_t nh = (size_t)B * 3 * H * dv * es, nvb = (size_t)B * H * dv * es;
    if (hist_in && overlap(hist_in, nh, hist_out, nh)) return JET_ERR_INVALID_ARG;
    if (overlap(v, nvb, o, nvb) || overlap(v, nvb, hist_out, nh) || overlap(o, nvb, hist_out, nh))
        return JET_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(o) || !aligned16(hist_out) || (hist_in && !aligned16(hist_in)))
        return JET_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the generator and the conv of the new tokens, with the history shift: v' goes to o,
    // which the update then reads (each element before the same thread overwrites it)
    st = dt == JET_BF16 ? launch_genconv<__nv_bfloat16>(x, w1, w2, v, hist_in, o, hist_out, taps, B, 1, D, H, dv, s)
                        : launch_genconv<float>(x, w1, w2, v, hist_in, o, hist_out, taps, B, 1, D, H, dv, s);
    if (st != JET_OK) return st;
    // that launch writes only v', the history and the taps: the update reads its state rows
    // and token vectors before it waits for it
    if (dt == JET_BF16)
        return dispatch_decode<__nv_bfloat16>(dk, q, k, o, g, beta, S, o, B, H, dv, s, nullptr, nullptr, 0, 1);
    return dispatch_decode<float>(dk, q, k, o, g, beta, S, o, B, H, dv, s, nullptr, nullptr, 0, 1);
}

jet_status jet_jetblock_decode_slots(const void* x, const void* w1, const void* w2, const void* q, const void* k,
                                     const void* v, const float* g, const float* beta, void* hist_pool,
                                     float* S_pool, const int* slots, int n_slots, void* o, void* v_conv,
                                     float* taps, int B, int D, int H, int dk, int dv, int hidden, int width,
                                     jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, 1, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!q || !k || !v || !g || !beta || !hist_pool || !S_pool || !slots || !o || !v_conv) return JET_ERR_INVALID_ARG;
    if (n_slots <= 0 || B > n_slots) return JET_ERR_INVALID_ARG;
    const long long nv = elems({B, H, dv});
    if (nv < 0 || elems({n_slots, H, dv, dk}) < 0 || elems({n_slots, 3, H, dv}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    const size_t es = esize(dt);
    for (const void* p : {q, k, (const void*)o})
        if (!aligned_to(p, es)) return JET_ERR_MISALIGNED;
    for (const void* p : {v, (const void*)v_conv, (const void*)hist_pool, (const void*)S_pool})
        if (!aligned16(p)) return JET_ERR_MISALIGNED;
    if (!aligned_to(g, 4) || !aligned_to(beta, 4) || !aligned_to(slots, 4) || (taps && !aligned_to(taps, 4)))
        return JET_ERR_MISALIGNED;
    if (overlap(v, (size_t)nv * es, v_conv, (size_t)nv * es)) return JET_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // generator + conv of the new tokens with the histories of their slots (updated in place)
    st = dt == JET_BF16 ? launch_genconv<__nv_bfloat16>(x, w1, w2, v, hist_pool, v_conv, hist_pool, taps, B, 1, D, H,
                                                       dv, s, slots, n_slots)
                        : launch_genconv<float>(x, w1, w2, v, hist_pool, v_conv, hist_pool, taps, B, 1, D, H, dv, s,
                                                slots, n_slots);
    if (st != JET_OK) return st;
    if (dt == JET_BF16)
        return dispatch_decode<__nv_bfloat16>(dk, q, k, v_conv, g, beta, S_pool, o, B, H, dv, s, nullptr, slots,
                                              n_slots, 1);
    return dispatch_decode<float>(dk, q, k, v_conv, g, beta, S_pool, o, B, H, dv, s, nullptr, slots, n_slots, 1);
}

jet_status jet_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return JET_ERR_CUDA;
    int word = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&word, jet::g_dev_error, sizeof(int)) != cudaSuccess) return JET_ERR_CUDA;
    if (cudaMemcpyToSymbol(jet::g_dev_error, &zero, sizeof(int)) != cudaSuccess) return JET_ERR_CUDA;
    if (word & DEVERR_TIMEOUT) return JET_ERR_TIMEOUT;
    if (word & DEVERR_DATA) return JET_ERR_DEVICE;
    return JET_OK;
}

const char* jet_status_string(jet_status s) {
    switch (s) {
        case JET_OK: return "JET_OK";
        case JET_ERR_INVALID_ARG: return "JET_ERR_INVALID_ARG";
        case JET_ERR_UNSUPPORTED: return "JET_ERR_UNSUPPORTED";
        case JET_ERR_MISALIGNED: return "JET_ERR_MISALIGNED";
        case JET_ERR_CUDA: return "JET_ERR_CUDA";
        case JET_ERR_TIMEOUT: return "JET_ERR_TIMEOUT";
        case JET_ERR_DEVICE: return "JET_ERR_DEVICE";
        case JET_ERR_WORKSPACE: return "JET_ERR_WORKSPACE";
        case JET_ERR_TOO_LARGE: return "JET_ERR_TOO_LARGE";
        case JET_ERR_LIBRARY: return "JET_ERR_LIBRARY";
    }
    return "JET_ERR_UNKNOWN";
}

uint64_t jet_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ---------------------------------------------------------------- prefill without a caller workspace
// Scratch for jet_gdn_prefill_noalloc: one fixed device array per GPU that
// loads this library (held until the process exits). Host code cannot use
// the array's name as a device address; the address is looked up per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[JET_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// per device: the context the address was looked up in, and the address
struct NoallocEntry { void* ctx; void* ptr; };
NoallocEntry g_noalloc[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (CtxGetCurrentFn) nullptr;
        return (CtxGetCurrentFn)p;
    }();
    return fn;
}

// Device address of the scratch array in the current device's current
// context. The address belongs to the context the module was loaded into, so
// it is cached together with that context and looked up again when the
// context changes (e.g. after cudaDeviceReset made a new primary context).
jet_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return JET_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return JET_ERR_UNSUPPORTED;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (!get_ctx) return JET_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return JET_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocEntry& e = g_noalloc[dev];
    if (ctx == nullptr || e.ptr == nullptr || e.ctx != (void*)ctx) {
        // set-up on this device: the lookup also makes the runtime's primary
        // context current if no context was yet (no allocation either way)
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return JET_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return JET_ERR_CUDA;
        e.ctx = (void*)ctx;
        e.ptr = p;
    }
    *out = e.ptr;
    return JET_OK;
}
}  // namespace

extern "C" jet_status jet_gdn_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                                              const float* beta, const float* S0, void* o, float* S_out, int B,
                                              int T, int H, int dk, int dv, int chunk, jet_dtype dt, void* stream) {
    // same argument checks as jet_gdn_prefill, before anything else
    if (!q || !k || !v || !g || !beta || !o || !S_out) return JET_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return JET_ERR_INVALID_ARG;
    if (elems({B, T, H, dk}) < 0 || elems({B, T, H, dv}) < 0 || elems({B, H, dv, dk}) < 0) return JET_ERR_INVALID_ARG;
    if (!shape_ok(dk, dv) || chunk != 64 || B > 65535 || H > 65535) return JET_ERR_UNSUPPORTED;
    // the fastest plan whose scratch fits the array
    const size_t need_min = jet_gdn_prefill_workspace_min(B, T, H, dk, dv, chunk, dt);
    if (need_min > (size_t)JET_NOALLOC_SCRATCH_BYTES) return JET_ERR_TOO_LARGE;
    const size_t need = jet_gdn_prefill_workspace_size(B, T, H, dk, dv, chunk, dt);
    const size_t use = need <= (size_t)JET_NOALLOC_SCRATCH_BYTES ? need : need_min;
    void* ws = nullptr;
    if (use > 0) {
        const jet_status st = noalloc_scratch(&ws);
        if (st != JET_OK) return st;
    }
    return jet_gdn_prefill(q, k, v, g, beta, S0, o, S_out, ws, use, B, T, H, dk, dv, chunk, dt, stream);
}


// ---- the JetBlock layer around the mixer (projections, gates, output gate and norm)
namespace {
// cuBLAS for the layer's plain GEMMs, loaded on first use (libjet.so itself
// does not depend on it); one handle per device
struct Blas {
    bool tried = false, ok = false;
    cublasStatus_t (*create)(cublasHandle_t*) = nullptr;
    cublasStatus_t (*set_stream)(cublasHandle_t, cudaStream_t) = nullptr;
    cublasStatus_t (*gemm_ex)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void*,
                              const void*, cudaDataType_t, int, const void*, cudaDataType_t, int, const void*, void*,
                              cudaDataType_t, int, cublasComputeType_t, cublasGemmAlgo_t) = nullptr;
    cublasHandle_t handle[64] = {};
};
std::mutex g_blas_mu;
Blas g_blas;

// under g_blas_mu: the loaded library and this device's handle bound to stream s
cublasHandle_t blas_handle(cudaStream_t s) {
    Blas& b = g_blas;
    if (!b.tried) {
        b.tried = true;
        void* lib = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
        if (!lib) lib = dlopen("libcublas.so", RTLD_NOW | RTLD_GLOBAL);
        if (lib) {
            b.create = reinterpret_cast<decltype(b.create)>(dlsym(lib, "cublasCreate_v2"));
            b.set_stream = reinterpret_cast<decltype(b.set_stream)>(dlsym(lib, "cublasSetStream_v2"));
            b.gemm_ex = reinterpret_cast<decltype(b.gemm_ex)>(dlsym(lib, "cublasGemmEx"));
            b.ok = b.create && b.set_stream && b.gemm_ex;
        }
    }
    if (!b.ok) return nullptr;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!b.handle[dev] && b.create(&b.handle[dev]) != CUBLAS_STATUS_SUCCESS) return nullptr;
    if (b.set_stream(b.handle[dev], s) != CUBLAS_STATUS_SUCCESS) return nullptr;
    return b.handle[dev];
}

// row-major C[M][N] = A[M][K] B[K][N] (bf16 A and B, float32 accumulate; C bf16 or float32)
jet_status gemm_rm(cublasHandle_t h, const void* A, const void* Bm, void* C, int M, int N, int K, bool c_f32) {
    const float one = 1.f, zero = 0.f;
    // column-major view: C^T[N][M] = B^T[N][K] A^T[K][M]
    const cublasStatus_t st = g_blas.gemm_ex(h, CUBLAS_OP_N, CUBLAS_OP_N, N, M, K, &one, Bm, CUDA_R_16BF, N, A,
                                             CUDA_R_16BF, K, &zero, C, c_f32 ? CUDA_R_32F : CUDA_R_16BF, N,
                                             CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return st == CUBLAS_STATUS_SUCCESS ? JET_OK : JET_ERR_CUDA;
}

struct LayerWs {       // byte offsets in the layer's workspace
    size_t q, k, v, z, g, b, o, mix, bytes;
};
LayerWs layer_ws(int B, int T, int H, int dk, int dv) {
    auto up = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    const size_t N = (size_t)B * T;
    LayerWs w;
    size_t off = 0;
    w.q = off; off += up(N * H * dk * 2);
    w.k = off; off += up(N * H * dk * 2);
    w.v = off; off += up(N * H * dv * 2);
    w.z = off; off += up(N * H * dv * 2);
    w.g = off; off += up(N * H * 4);
    w.b = off; off += up(N * H * 4);
    w.o = off; off += up(N * H * dv * 2);
    w.mix = off;
    const size_t mix = T == 1 ? up((size_t)B * H * 4 * sizeof(float))
                              : jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, 64, JET_BF16);
    w.bytes = off + mix;
    return w;
}
}  // namespace

size_t jet_jetblock_layer_workspace_size(int B, int T, int D, int H, int dk, int dv) {
    if (B <= 0 || T <= 0 || D <= 0 || H <= 0 || D % 16 != 0 || !tc_prefill_ok(JET_BF16, dk, dv, (long long)B * T))
        return 0;
    if (elems({B, T, H, dv}) < 0 || elems({B, T, D}) < 0) return 0;
    return layer_ws(B, T, H, dk, dv).bytes;
}

jet_status jet_jetblock_layer(const void* x, const void* wq, const void* wk, const void* wv, const void* wg,
                              const void* wb, const void* wz, const void* wo, const float* gamma, const void* w1,
                              const void* w2, const void* hist_in, void* hist_out, const float* S0, float* S_out,
                              void* y, void* workspace, size_t ws_bytes, int B, int T, int D, int H, int dk, int dv,
                              int hidden, int width, jet_dtype dt, void* stream) {
    jet_status st = check_gen(x, w1, w2, B, T, D, H, hidden, width, dt);
    if (st != JET_OK) return st;
    if (!wq || !wk || !wv || !wg || !wb || !wz || !wo || !gamma || !S_out || !y) return JET_ERR_INVALID_ARG;
    if (elems({B, T, H, dv}) < 0 || elems({B, T, H, dk}) < 0 || elems({D, H, dv}) < 0 ||
        elems({B, H, dv, dk}) < 0)
        return JET_ERR_INVALID_ARG;
    if (dt != JET_BF16 || !tc_prefill_ok(dt, dk, dv, (long long)B * T) || B > 65535 || H > 65535)
        return JET_ERR_UNSUPPORTED;
    for (const void* p : {wq, wk, wv, wg, wb, wz, wo, hist_in, (const void*)hist_out, (const void*)y})
        if (p && !aligned_to(p, 2)) return JET_ERR_MISALIGNED;
    for (const void* p : {hist_in, (const void*)hist_out, (const void*)S0, (const void*)S_out, (const void*)gamma,
                          (const void*)workspace})
        if (p && !aligned16(p)) return JET_ERR_MISALIGNED;
    if (T == 1 && !hist_out) return JET_ERR_INVALID_ARG;      // a decode step shifts the history
    if (!workspace) ws_bytes = 0;
    const LayerWs L = layer_ws(B, T, H, dk, dv);
    if (ws_bytes < L.bytes) return JET_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    auto* q = w + L.q;
    auto* k = w + L.k;
    auto* v = w + L.v;
    auto* z = w + L.z;
    float* g = reinterpret_cast<float*>(w + L.g);
    float* b = reinterpret_cast<float*>(w + L.b);
    auto* o = w + L.o;
    const int N = B * T;
    {   // the projections (plain GEMMs on cuBLAS)
        std::lock_guard<std::mutex> lk(g_blas_mu);
        cublasHandle_t h = blas_handle(s);
        if (!h) return g_blas.ok ? JET_ERR_CUDA : JET_ERR_LIBRARY;
        for (auto [wm, out, cols, f32] : {std::tuple<const void*, void*, int, bool>{wq, q, H * dk, false},
                                          {wk, k, H * dk, false}, {wv, v, H * dv, false}, {wz, z, H * dv, false},
                                          {wg, g, H, true}, {wb, b, H, true}}) {
            st = gemm_rm(h, x, wm, out, N, cols, D, f32);
            if (st != JET_OK) return st;
        }
    }
    const long long nh = (long long)N * H;
    st = launch(layer::gates_kernel, dim3((unsigned)std::min<long long>((nh + 255) / 256, 4096)),
                dim3(layer::GATE_THREADS), 0, s, g, b, nh);
    if (st != JET_OK) return st;
    // the mixer
    if (T == 1) {     // one new token per sequence: S advanced in place in S_out
        if (S0 != S_out) {
            const cudaError_t e = S0 ? cudaMemcpyAsync(S_out, S0, sizeof(float) * (size_t)B * H * dv * dk,
                                                       cudaMemcpyDeviceToDevice, s)
                                     : cudaMemsetAsync(S_out, 0, sizeof(float) * (size_t)B * H * dv * dk, s);
            if (e != cudaSuccess) return JET_ERR_CUDA;
        }
        float* taps = reinterpret_cast<float*>(w + L.mix);
        st = launch_genconv<__nv_bfloat16>(x, w1, w2, v, hist_in, o, hist_out, taps, B, 1, D, H, dv, s);
        if (st != JET_OK) return st;
        st = dispatch_decode<__nv_bfloat16>(dk, q, k, o, g, b, S_out, o, B, H, dv, s, nullptr, nullptr, 0, 1);
    } else {
        st = jet_jetblock_prefill(x, w1, w2, q, k, v, hist_in, hist_out, g, b, S0, o, S_out, w + L.mix,
                                  ws_bytes - L.mix, B, T, D, H, dk, dv, hidden, width, 64, dt, stream);
    }
    if (st != JET_OK) return st;
    // per-head RMSNorm, gamma and the SiLU output gate (in place over o), then the output projection
    const long long rows = (long long)N * H;
    const unsigned grid = (unsigned)((rows + layer::OUT_THREADS / 32 - 1) / (layer::OUT_THREADS / 32));
    st = dv <= 256 ? launch(layer::out_gate_kernel<1>, dim3(grid), dim3(layer::OUT_THREADS), 0, s,
                            (const __nv_bfloat16*)o, (const __nv_bfloat16*)z, gamma, (__nv_bfloat16*)o, rows, dv)
                   : launch(layer::out_gate_kernel<2>, dim3(grid), dim3(layer::OUT_THREADS), 0, s,
                            (const __nv_bfloat16*)o, (const __nv_bfloat16*)z, gamma, (__nv_bfloat16*)o, rows, dv);
    if (st != JET_OK) return st;
    std::lock_guard<std::mutex> lk(g_blas_mu);
    cublasHandle_t h = blas_handle(s);
    if (!h) return JET_ERR_CUDA;
    return gemm_rm(h, o, wo, y, N, D, H * dv, false);
}

#ifdef JET_TEST_WAIT_EXPIRY
// test builds only: see g_test_skip_p2a
extern "C" int jet_test_skip_p2a(int on) {
    return cudaMemcpyToSymbol(jet::pfch::g_test_skip_p2a, &on, sizeof(int)) == cudaSuccess ? 0 : 1;
}
#endif
