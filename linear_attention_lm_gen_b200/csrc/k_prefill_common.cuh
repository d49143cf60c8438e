// Shared pieces of the chunked Gated DeltaNet prefill kernels (sm_100a):
// the per-chunk preparation that does not depend on the state (Jet-Nemotron
// paper, section 2.3, gated delta rule in chunked WY / UT form), written as
// device functions used both by the fused kernel (which prepares chunk c+1
// while the state chain runs chunk c) and by the stand-alone preparation
// kernel (which prepares every chunk of every sequence at once).
//
// For a chunk of C = 64 tokens (r, i index tokens):
//   G_r = sum_{t<=r} g_t (kept in log2 units),  gam_r = exp(G_r)
//   d_i = exp(G_{L-1} - G_i) (0 past the chunk end L)
//   A_ri = b_r exp(G_r - G_i) k^_r.k^_i (i < r),  P_ri = exp(G_r - G_i) q^_r.k^_i (i <= r)
//   T = (I + A)^-1,  T1 = T diag(b),  T2 = T diag(b gam / |k|)
//   Q~ = diag(gam / |q|) Q,  W^T = K^T T2^T
// The functions are called by a group of 256 threads (8 warps, index pt) that
// synchronise on named barrier `bid`; TMEM reads follow the lane-quarter rule
// (warp pw reads lanes 32 (pw & 3) .. +31).
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "sm100.cuh"

namespace jet {
namespace pfws {

using namespace sm100;

constexpr int C = 64;
constexpr int ROWS = 128;                              // state rows per CTA (TMEM lanes)
constexpr int NPREP = 256;                             // threads of a preparation group
constexpr float EPS = 1e-6f;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int LDA = 68;                                // fp32 row stride of A / T
constexpr int LDX = 40;                                // row stride of the 32 x 32 block products
constexpr int LDX1 = 24;                               // row stride of the 16 x 16 block products
constexpr uint32_t AF_BYTES = 64 * LDA * 4;            // A / T scratch
// row stride (floats) of a segment transition A_p [dk][dk] in the workspace:
// padded so that the combine's tensor-core fragment loads hit distinct banks
__host__ __device__ constexpr int trans_ld(int dk) { return dk + 8; }
constexpr uint32_t XS_BYTES = 32 * LDX * 4;            // block-product scratch

struct Vec {       // per-token vectors of one chunk (64 floats each)
    float* G;      // cumulative gate, log2 units
    float* gam;    // exp(G)
    float* dcy;    // exp(G_{L-1} - G_i), 0 past the chunk end
    float* bet;
    float* ik;     // 1/|k|
    float* iq;     // 1/|q|
    float* graw;
    float* F;      // exp(G_31 - G_i) for i < 32 (the lower-left block factor)
};
__device__ __forceinline__ Vec vec_from(float* v) {    // 8 x 64 floats
    return Vec{v, v + 64, v + 128, v + 192, v + 256, v + 320, v + 384, v + 448};
}

// 2^x via the MUFU ex2 instruction (relative error ~2^-22; results below
// 2^-126 flush to zero, which only ever affects decays that are negligible)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory");
}

// bounded wait that also gives up when another thread raised the abort flag
// (a short sleep between polls keeps idle waiters from taking issue slots
// from the warps that are computing); on running out of time it raises the
// abort flag itself and sets the device error word
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255u) == 255u) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > kWaitLimitNs) break;
        }
        __nanosleep(64);
    }
    *abort_flag = 1;
    flag_error(DEVERR_TIMEOUT);
    return false;
}
// true on every thread of named barrier `id` iff `ok` holds on all of them
__device__ __forceinline__ bool group_all(int id, int n, bool ok) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
        " bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r) : "r"((uint32_t)ok), "r"(id), "r"(n) : "memory");
    return r != 0;
}
__device__ __forceinline__ void arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
    return make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
}
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
// warp-level m16n8k8 tf32 MMA (float32 accumulate); operands rounded to tf32
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D[16 x 8] += A[16 x 8k] B[8k x 8] over ksteps steps of 8; A and B in shared
// memory (row strides lda, ldb); fragment layout of m16n8k8: lane = 4 g + t,
// A rows g, g+8 / cols t, t+4; B rows t, t+4 / col g; D rows g, g+8 / cols 2t, 2t+1
__device__ __forceinline__ void warp_mm_tf32(float* d, const float* A, int lda, const float* B, int ldb,
                                             int ksteps, int lane) {
    const int g = lane >> 2, t = lane & 3;
    for (int ks = 0; ks < ksteps; ++ks) {
        const float* a = A + ks * 8;
        const float* bb = B + ks * 8 * ldb;
        mma_tf32(d, to_tf32(a[g * lda + t]), to_tf32(a[(g + 8) * lda + t]), to_tf32(a[g * lda + t + 4]),
                 to_tf32(a[(g + 8) * lda + t + 4]), to_tf32(bb[t * ldb + g]), to_tf32(bb[(t + 4) * ldb + g]));
    }
}
// byte offset of 16-byte chunk `ch` (8 bf16 columns) of row `r` in a K/Q tile
// stored as 64-column SW128 blocks of stride `bstride`
__device__ __forceinline__ uint32_t blk_chunk(int r, int ch, uint32_t bstride) {
    return (uint32_t)(ch >> 3) * bstride + sw128_off((uint32_t)r, (uint32_t)(ch & 7) * 16u);
}

// Segment decomposition of the token axis (sequence parallelism; the
// recurrence is affine in the state, S_end = S_start A + B, so segments can
// run concurrently once their start states are known):
//   phase A  every segment p < P-1 runs from a zero state (p > 0) or S0
//            (p = 0) and writes its end state B_p; an extra 128-row slice
//            starts from the identity with zero values and yields the
//            segment's dk x dk transition A_p;
//   combine  S_start(p+1) = S_start(p) A_p + B_p (seg_combine_kernel);
//   phase C  every segment runs from its true start state and writes o; the
//            last one writes the final state.
// P = 1 is the plain single pass.
struct Seg {
    int nseg;          // P
    int seg_chunks;    // chunks per segment (the last may be shorter)
    int zseg;          // segments covered by this launch (blockIdx.z = b * zseg + p)
    int phaseA;        // 1: end states and transitions, no outputs
    const float* Sst;  // phase C start states (P > 1): [B][P][H][dv][dk]
    float* Eo;         // phase A end states: [B][P-1][H][dv][dk]
    float* Ao;         // phase A transitions: [B][P-1][H][dk][trans_ld(dk)]
};


// Variable-length batches (one launch over sequences of different lengths,
// packed along the token axis): sequence i holds tokens tok[i] .. tok[i+1]-1,
// chunks chunk[i] .. chunk[i+1]-1 of the per-chunk buffers (images, output
// corrections) and segments seg[i] .. seg[i+1]-1 (all segments seg_chunks
// long but the last of a sequence). The table rides in the kernel parameters,
// so no device-side copy is needed. nseq == 0: the dense layout, B sequences
// of Tn tokens, located by arithmetic.
constexpr int kMaxVarlenSeqs = 256;
struct SeqMap {
    int nseq;
    int seg_chunks;
    int tok[kMaxVarlenSeqs + 1];
    int chunk[kMaxVarlenSeqs + 1];
    int seg[kMaxVarlenSeqs + 1];
};
// the sequence i with off[i] * mul <= x < off[i + 1] * mul (off increasing, off[0] = 0)
__device__ __forceinline__ int seq_of(const int* off, int nseq, long long x, int mul) {
    int lo = 0, hi = nseq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((long long)off[mid] * mul <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One preparation item = one (sequence, head, chunk); item index = image index:
// dense (b H + h) nct + c, variable-length chunk[i] H + h nct_i + c.
struct ItemInfo {
    int z;        // first token row of the chunk in the token axis
    int c;        // chunk within its sequence
    int h;        // head
    int L;        // tokens of the chunk (64, or fewer at the sequence end)
};
__device__ __forceinline__ ItemInfo item_info(int item, int Tn, int H, int nct, const SeqMap& sq) {
    ItemInfo r;
    if (sq.nseq == 0) {
        r.c = item % nct;
        r.h = (item / nct) % H;
        const int b = item / nct / H;
        r.z = b * Tn + r.c * C;
        r.L = min(C, Tn - r.c * C);
    } else {
        const int i = seq_of(sq.chunk, sq.nseq, item, H);
        const int nci = sq.chunk[i + 1] - sq.chunk[i], rr = item - sq.chunk[i] * H;
        r.h = rr / nci;
        r.c = rr % nci;
        r.z = sq.tok[i] + r.c * C;
        r.L = min(C, sq.tok[i + 1] - r.z);
    }
    return r;
}

// ---------------------------------------------------------------- preparation steps

// Per-token vectors of one chunk: records g and b (gb: g for pt < 64, b for
// 64 <= pt < 128, 0 past the chunk end), the inverse L2 norms of the k and q
// rows of the K/Q tile (64-column blocks [K 8K | Q 8K] of stride 16K), the
// cumulative gates, gam, d and the lower-left block factor F.
template <int DK>
__device__ __forceinline__ void prep_vectors(const uint8_t* KQ, Vec V, float* PN, float gb, int L, int pt, int bid) {
    constexpr int NCH = DK / 8;
    const int pw = pt >> 5, lane = pt & 31;
    if (pt < 64) V.graw[pt] = gb; else if (pt < 128) V.bet[pt - 64] = gb;
    {   // L2 norms: row = pt & 127 (k rows then q rows), half of the columns
        const int row = pt & 127, half = pt >> 7;
        const uint32_t qoff = row < 64 ? 0u : 8192u;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < NCH / 2; ++j) {
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(KQ + qoff + blk_chunk(row & 63, half * (NCH / 2) + j, 16384)), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
        }
        PN[half * 128 + row] = ss;
    }
    named_sync(bid, NPREP);
    if (pt < 128) {
        const float inv = 1.0f / sqrtf(PN[pt] + PN[128 + pt] + EPS);
        if (pt < 64) V.ik[pt] = inv; else V.iq[pt - 64] = inv;
    }
    if (pw == 0) {   // inclusive scan of the gates, two per lane, in log2 units
        const float a0 = V.graw[2 * lane], a1 = a0 + V.graw[2 * lane + 1];
        float run = a1;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, run, o2);
            if (lane >= o2) run += y;
        }
        V.G[2 * lane] = (run - a1 + a0) * LOG2E;
        V.G[2 * lane + 1] = run * LOG2E;
    }
    named_sync(bid, NPREP);
    if (pt < 64) {
        V.gam[pt] = fast_exp2(V.G[pt]);
        V.dcy[pt] = pt < L ? fast_exp2(V.G[L - 1] - V.G[pt]) : 0.f;
    } else if (pt < 96) {
        V.F[pt - 64] = fast_exp2(V.G[31] - V.G[pt - 64]);
    }
    named_sync(bid, NPREP);
}

// A (fp32, into AF) and P (bf16 SW128 tile Pt) from the P1 product
// [K; Q] K^T held in TMEM columns xp .. xp+63 (rows 0-63: K K^T, 64-127: Q K^T).
// No barrier inside; the caller synchronises before AF is read.
__device__ __forceinline__ void prep_e1(uint32_t xp, Vec V, float* AF, uint8_t* Pt, int pt) {
    const int pw = pt >> 5, lane = pt & 31;
    const int q4 = pw & 3, hh = pw >> 2;                 // TMEM lane quarter, column half
    uint32_t x[32];
    tmem_ld32(xp + ((uint32_t)(q4 * 32) << 16) + hh * 32, x);
    tmem_ld_wait();
    const int rb = q4 & 1;                               // 32-row block of the thread's row
    const int r = rb * 32 + lane;
    const float Gr = V.G[r];
    // lower-left block (rb = 1, hh = 0): exp(G_r - G_i) = exp(G_r - G_31) exp(G_31 - G_i),
    // both factors <= 1; upper-right block (rb = 0, hh = 1) is all zero (i > r)
    const bool zero_blk = rb == 0 && hh == 1;
    const bool fact_blk = rb == 1 && hh == 0;
    const float Rr = fact_blk ? fast_exp2(Gr - V.G[31]) : 0.f;
    const float4* G4 = reinterpret_cast<const float4*>(V.G + hh * 32);
    const float4* K4 = reinterpret_cast<const float4*>(V.ik + hh * 32);
    const float4* F4 = reinterpret_cast<const float4*>(V.F);
    float e[32];
#pragma unroll
    for (int i4 = 0; i4 < 8; ++i4) {
        const float4 gg = G4[i4], kk = K4[i4];
        const float gv[4] = {gg.x, gg.y, gg.z, gg.w}, kv[4] = {kk.x, kk.y, kk.z, kk.w};
        float fv[4] = {0.f, 0.f, 0.f, 0.f};
        if (fact_blk) { const float4 ff = F4[i4]; fv[0] = ff.x; fv[1] = ff.y; fv[2] = ff.z; fv[3] = ff.w; }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = i4 * 4 + u;
            const float dec = zero_blk ? 0.f : (fact_blk ? Rr * fv[u] : fast_exp2(Gr - gv[u]));
            e[j] = dec * __uint_as_float(x[j]) * kv[u];
        }
    }
    if (q4 < 2) {
        const float sc = V.bet[r] * V.ik[r];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
            const int i = hh * 32 + i4 * 4;
            float4 a;
            a.x = i + 0 < r ? sc * e[i4 * 4 + 0] : 0.f;
            a.y = i + 1 < r ? sc * e[i4 * 4 + 1] : 0.f;
            a.z = i + 2 < r ? sc * e[i4 * 4 + 2] : 0.f;
            a.w = i + 3 < r ? sc * e[i4 * 4 + 3] : 0.f;
            *reinterpret_cast<float4*>(AF + r * LDA + i) = a;
        }
    } else {
        const float sc = V.iq[r];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = hh * 32 + ch * 8 + u;
                f[u] = i <= r ? sc * e[ch * 8 + u] : 0.f;
            }
            *reinterpret_cast<uint4*>(Pt + sw128_off(r, (hh * 32 + ch * 8) * 2)) = pack8(f);
        }
    }
}

// T = (I + A)^-1 in place in AF (A strictly lower triangular): 16 x 16
// diagonal blocks by forward substitution, then 16 -> 32 -> 64 doubling with
// tf32 warp MMAs. Starts and ends with a barrier-complete AF.
__device__ __forceinline__ void ut_inverse(float* AF, float* XS, int pt, int bid) {
    const int pw = pt >> 5, lane = pt & 31;
    float t[16];
    if (pt < 64) {
        const int cc = pt, j = cc >> 4, cl = cc & 15;
        const float* Ab = AF + (j * 16) * LDA + j * 16;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float xv = (r == cl) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) xv -= Ab[r * LDA + i] * t[i];
            t[r] = xv;
        }
    }
    named_sync(bid, NPREP);
    if (pt < 64) {
        const int cc = pt, j = cc >> 4;
#pragma unroll
        for (int r = 0; r < 16; ++r) AF[(j * 16 + r) * LDA + cc] = t[r];
    }
    named_sync(bid, NPREP);
    // 16 -> 32 for pairs (1,0) and (3,2): X = A_10 T_00, T_10 = -T_11 X
    // (warps 0-3: pair = pw >> 1, 8-column half = pw & 1)
    const int g8 = lane >> 2, t4 = lane & 3;
    if (pw < 4) {
        const int pr = pw >> 1, nh = pw & 1;
        const int b0 = pr * 2, b1 = b0 + 1;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm_tf32(d, AF + (b1 * 16) * LDA + b0 * 16, LDA, AF + (b0 * 16) * LDA + b0 * 16 + nh * 8, LDA, 2, lane);
        float* xo = XS + pr * 16 * LDX1 + nh * 8;
        xo[g8 * LDX1 + 2 * t4] = d[0];
        xo[g8 * LDX1 + 2 * t4 + 1] = d[1];
        xo[(g8 + 8) * LDX1 + 2 * t4] = d[2];
        xo[(g8 + 8) * LDX1 + 2 * t4 + 1] = d[3];
    }
    named_sync(bid, NPREP);
    if (pw < 4) {
        const int pr = pw >> 1, nh = pw & 1;
        const int b0 = pr * 2, b1 = b0 + 1;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm_tf32(d, AF + (b1 * 16) * LDA + b1 * 16, LDA, XS + pr * 16 * LDX1 + nh * 8, LDX1, 2, lane);
        float* to = AF + (b1 * 16) * LDA + b0 * 16 + nh * 8;
        to[g8 * LDA + 2 * t4] = -d[0];
        to[g8 * LDA + 2 * t4 + 1] = -d[1];
        to[(g8 + 8) * LDA + 2 * t4] = -d[2];
        to[(g8 + 8) * LDA + 2 * t4 + 1] = -d[3];
    }
    named_sync(bid, NPREP);
    // 32 -> 64: X = A[32:64][0:32] T[0:32][0:32], T[32:64][0:32] = -T[32:64][32:64] X
    // (warp pw: 16-row half mt = pw >> 2, 8-column quarter nq = pw & 3)
    {
        const int mt = pw >> 2, nq = pw & 3;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm_tf32(d, AF + (32 + mt * 16) * LDA, LDA, AF + nq * 8, LDA, 4, lane);
        float* xo = XS + (mt * 16) * LDX + nq * 8;
        xo[g8 * LDX + 2 * t4] = d[0];
        xo[g8 * LDX + 2 * t4 + 1] = d[1];
        xo[(g8 + 8) * LDX + 2 * t4] = d[2];
        xo[(g8 + 8) * LDX + 2 * t4 + 1] = d[3];
    }
    named_sync(bid, NPREP);
    {
        const int mt = pw >> 2, nq = pw & 3;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        warp_mm_tf32(d, AF + (32 + mt * 16) * LDA + 32, LDA, XS + nq * 8, LDX, 4, lane);
        float* to = AF + (32 + mt * 16) * LDA + nq * 8;
        to[g8 * LDA + 2 * t4] = -d[0];
        to[g8 * LDA + 2 * t4 + 1] = -d[1];
        to[(g8 + 8) * LDA + 2 * t4] = -d[2];
        to[(g8 + 8) * LDA + 2 * t4 + 1] = -d[3];
    }
    named_sync(bid, NPREP);
}

// T1 = T diag(b) and T2 = T diag(b gam / |k|) as bf16 SW128 tiles (row r = pt >> 2,
// 16 columns per thread; T1 skipped when null). No barrier inside.
__device__ __forceinline__ void prep_t1t2(const float* AF, Vec V, uint8_t* T1, uint8_t* T2, int pt) {
    const int r = pt >> 2, qc = pt & 3;
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
        const int i0 = qc * 16 + hc * 8;
        float f1[8], f2[8];
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
            const float4 tv = *reinterpret_cast<const float4*>(AF + r * LDA + i0 + h4 * 4);
            const float4 bv = *reinterpret_cast<const float4*>(V.bet + i0 + h4 * 4);
            const float4 gv = *reinterpret_cast<const float4*>(V.gam + i0 + h4 * 4);
            const float4 kv = *reinterpret_cast<const float4*>(V.ik + i0 + h4 * 4);
            const float t_[4] = {tv.x, tv.y, tv.z, tv.w}, b_[4] = {bv.x, bv.y, bv.z, bv.w};
            const float g_[4] = {gv.x, gv.y, gv.z, gv.w}, k_[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = i0 + h4 * 4 + e;
                const float t1v = i <= r ? t_[e] * b_[e] : 0.f;
                f1[h4 * 4 + e] = t1v;
                f2[h4 * 4 + e] = t1v * g_[e] * k_[e];
            }
        }
        const uint32_t off = sw128_off(r, i0 * 2);
        if (T1) *reinterpret_cast<uint4*>(T1 + off) = pack8(f1);
        *reinterpret_cast<uint4*>(T2 + off) = pack8(f2);
    }
}

// float4 slot of token i's taps in a shared-memory taps array: one slot of
// padding after every 16 tokens, so the four 16-token column groups of
// prep_t1t2_conv read distinct banks
__host__ __device__ constexpr int tp_slot(int i) { return i + (i >> 4); }
constexpr uint32_t TP_BYTES = 68 * 16;

// prep_t1t2 with the dynamic causal conv of the chunk's values folded into T1
// (Jet-Nemotron paper, section 2.4: v'_i = sum_j w_i[j] v_{i-j}). U = T1 V' is
// linear in the raw values, U = M V + MH V_prev, where
//   M[r][s]  = sum_{j=0..3} w_{s+j}[j] T1[r][s+j]        (s = 0..63; T1[r][i] = 0 for i > r)
//   MH[r][s] = sum_{j=-s..3} w_{s+j}[j] T1[r][s+j]        (s = -3..-1: the previous chunk's last tokens)
// TP: the chunk's taps w_i (float4 at tp_slot(i), zero past the chunk end).
// M is stored where T1 would be (K-major SW128, rows r); MH as the K x N =
// 16 x 64 operand of one more K-step, MN-major SW128 (row 16 + s holds
// MH[.][s], rows 0..12 zero), all zero when `halo` is false (a sequence
// start with no history). T2 as in prep_t1t2. Row r = pt >> 2, 16 columns
// per thread; the three T1 values past them come from the next lane (same
// row). No barrier inside.
__device__ __forceinline__ void prep_t1t2_conv(const float* AF, Vec V, const float4* TP, uint8_t* M, uint8_t* MH,
                                               uint8_t* T2, bool halo, int pt) {
    const int r = pt >> 2, qc = pt & 3, i0 = qc * 16;
    float t1[19];                                        // T1[r][i0 .. i0+18]
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
        const int j0 = i0 + hc * 8;
        float f2[8];
#pragma unroll
        for (int h4 = 0; h4 < 2; ++h4) {
            const float4 tv = *reinterpret_cast<const float4*>(AF + r * LDA + j0 + h4 * 4);
            const float4 bv = *reinterpret_cast<const float4*>(V.bet + j0 + h4 * 4);
            const float4 gv = *reinterpret_cast<const float4*>(V.gam + j0 + h4 * 4);
            const float4 kv = *reinterpret_cast<const float4*>(V.ik + j0 + h4 * 4);
            const float t_[4] = {tv.x, tv.y, tv.z, tv.w}, b_[4] = {bv.x, bv.y, bv.z, bv.w};
            const float g_[4] = {gv.x, gv.y, gv.z, gv.w}, k_[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = j0 + h4 * 4 + e;
                const float t1v = i <= r ? t_[e] * b_[e] : 0.f;
                t1[hc * 8 + h4 * 4 + e] = t1v;
                f2[h4 * 4 + e] = t1v * g_[e] * k_[e];
            }
        }
        *reinterpret_cast<uint4*>(T2 + sw128_off(r, j0 * 2)) = pack8(f2);
    }
#pragma unroll
    for (int u = 0; u < 3; ++u) {
        const float nx = __shfl_down_sync(0xffffffffu, t1[u], 1);   // T1[r][i0 + 16 + u] (lane + 1: qc + 1)
        t1[16 + u] = qc < 3 ? nx : 0.f;
    }
    float m[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) m[u] = 0.f;
#pragma unroll
    for (int u = 0; u < 19; ++u) {                       // token i = i0 + u feeds M[r][i - j] through tap j
        const int i = i0 + u;
        const float4 w = i < C ? TP[tp_slot(i)] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float wj[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (u - j >= 0 && u - j < 16) m[u - j] = fmaf(wj[j], t1[u], m[u - j]);
    }
#pragma unroll
    for (int hc = 0; hc < 2; ++hc)
        *reinterpret_cast<uint4*>(M + sw128_off(r, (i0 + hc * 8) * 2)) = pack8(m + hc * 8);
    if (qc == 0) {                                       // MH[r][-3..-1] from T1[r][0..2] and w_0..w_2
        const float4 w0 = TP[tp_slot(0)], w1 = TP[tp_slot(1)], w2 = TP[tp_slot(2)];
        const float h1 = halo ? fmaf(w2.w, t1[2], fmaf(w1.z, t1[1], w0.y * t1[0])) : 0.f;   // s = -1
        const float h2 = halo ? fmaf(w1.w, t1[1], w0.z * t1[0]) : 0.f;                        // s = -2
        const float h3 = halo ? w0.w * t1[0] : 0.f;                                           // s = -3
        *reinterpret_cast<__nv_bfloat16*>(MH + sw128_off(13, r * 2)) = __float2bfloat16_rn(h3);
        *reinterpret_cast<__nv_bfloat16*>(MH + sw128_off(14, r * 2)) = __float2bfloat16_rn(h2);
        *reinterpret_cast<__nv_bfloat16*>(MH + sw128_off(15, r * 2)) = __float2bfloat16_rn(h1);
    }
    if (pt < 13 * 8)                                     // rows 0..12: zero (whole rows, layout-free)
        *reinterpret_cast<uint4*>(MH + pt * 16) = make_uint4(0u, 0u, 0u, 0u);
}

// Q~ = diag(gam / |q|) Q in place, Q the second half of each 64-column block
// of the K/Q tile. No barrier inside.
template <int DK>
__device__ __forceinline__ void prep_qtilde(uint8_t* KQ, Vec V, int pt) {
    constexpr int NCH = DK / 8;
    const int r = pt >> 2, qc = pt & 3;
    const float sq = V.gam[r] * V.iq[r];
#pragma unroll
    for (int j = qc; j < NCH; j += 4) {
        uint4* pq = reinterpret_cast<uint4*>(KQ + 8192 + blk_chunk(r, j, 16384));
        float f[8];
        unpack8(*pq, f);
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] *= sq;
        *pq = pack8(f);
    }
}

// W^T (rows = key features, 64 token columns) from the P2b product held in
// TMEM columns xw .. xw+63, as a bf16 SW128 tile. No barrier inside.
template <int DK>
__device__ __forceinline__ void prep_wt(uint32_t xw, uint8_t* WT, int pt) {
    const int pw = pt >> 5, lane = pt & 31;
    const int q4 = pw & 3, hh = pw >> 2;
    uint32_t x[32];
    tmem_ld32(xw + ((uint32_t)(q4 * 32) << 16) + hh * 32, x);
    tmem_ld_wait();
    const int j = q4 * 32 + lane;
    if (j < DK) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = __uint_as_float(x[ch * 8 + u]);
            *reinterpret_cast<uint4*>(WT + sw128_off(j, (hh * 32 + ch * 8) * 2)) = pack8(f);
        }
    }
}

}  // namespace pfws
}  // namespace jet
