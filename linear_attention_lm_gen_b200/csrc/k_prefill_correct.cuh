// Output correction of the one-pass sequence-parallel prefill.
//
// The chunked gated delta rule (Jet-Nemotron paper, section 2.3) gives a
// chunk's outputs as an affine function of the state S_c at the chunk start:
//   O_c = (Q~ - P W) S_c^T + P U.
// Inside a segment that started from a zero state instead of its true start
// state S*, the state at chunk c differs by S* Phi_c (Phi_c: the product of
// the transitions since the segment start), so the true outputs are
//   O_c = O0_c + Qe_c S*^T,   Qe_c = (Q~ - P W) Phi_c^T   [64 tokens x dk],
// where O0_c are the outputs the segment pass wrote and Qe_c is what its
// transition slice wrote. This kernel adds Qe_c S*^T for every chunk of the
// segments p >= 1.
//
// One CTA per (sequence, head, chunk): a 64 x dv by dk product on the tensor
// cores (bf16 mma.sync m16n8k16, float32 accumulate; 2 x 1.6 Mflop per chunk
// is far too small a tile for tcgen05, and the kernel is bound by moving the
// 32 KB output tile). The Qe tile, S* (in bf16, as the segment combine wrote
// it) and the output tile are copied into shared memory by 16-byte cp.async
// all at once (padded rows: conflict-free ldmatrix), then the output is
// written back with 16-byte stores. Warp w owns output columns
// [w dv/8, (w+1) dv/8).
#pragma once
#include "common.cuh"
#include "k_prefill_common.cuh"

namespace jet {
namespace pfcor {

constexpr int THREADS = 256;
constexpr int C = 64;

__host__ __device__ constexpr int lda(int dk) { return dk + 8; }      // bf16 row stride of Qe and S*
__host__ __device__ constexpr int ldo(int dv) { return dv + 8; }      // bf16 row stride of the output tile
__host__ __device__ constexpr size_t smem_bytes(int dk, int dv) {
    return 2 * ((size_t)C * lda(dk) + (size_t)dv * lda(dk) + (size_t)C * ldo(dv));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 :: "r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Dense: Qe [B][H][nct][64][DK] bf16; Sb [B][P][H][dv][DK] bf16 (the start
// state of the segment of chunk gc is entry gc / seg_chunks); o [B*T][H][dv]
// bf16 (updated in place). Chunks chunk0 .. nct-1; grid (nct - chunk0, H, B).
// Variable length (sq.nseq > 0): blockIdx.x runs over every chunk of every
// sequence (grid (total chunks, H, 1)); chunks of a sequence's first segment
// have nothing to add; Qe, Sb and the token rows follow the sequence map.
template <int DK, int DV>
__global__ void __launch_bounds__(THREADS)
prefill_correct_kernel(const __nv_bfloat16* __restrict__ Qe, const __nv_bfloat16* __restrict__ Sb,
                       __nv_bfloat16* __restrict__ o, int Tn, int H, int nct, int chunk0, int seg_chunks, int P,
                       const __grid_constant__ pfws::SeqMap sq) {
    static_assert(DK % 16 == 0 && DK <= 128 && DV % 64 == 0 && DV <= 256, "shapes");
    constexpr int LDA = lda(DK), LDO = ldo(DV);
    constexpr int NT = DV / 64;                    // n8 tiles per warp (DV / 8 columns)
    constexpr int KS = DK / 16;
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem);          // [64][LDA]
    __nv_bfloat16* ss = qs + C * LDA;                                    // [DV][LDA]
    __nv_bfloat16* os = ss + DV * LDA;                                   // [64][LDO]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y;
    // the chunk's index within its sequence, its Qe entry, its S* entry and its first token row
    int gc, L;
    long long qe_idx, sb_idx, row0;
    if (sq.nseq == 0) {
        const int b = blockIdx.z;
        gc = chunk0 + blockIdx.x;
        if (gc >= nct) return;
        const int p = gc / seg_chunks;
        qe_idx = ((long long)b * H + h) * nct + gc;
        sb_idx = ((long long)b * P + p) * H + h;
        row0 = (long long)b * Tn + (long long)gc * C;
        L = min(C, Tn - gc * C);
    } else {
        const int x = blockIdx.x;
        const int i = pfws::seq_of(sq.chunk, sq.nseq, x, 1);
        gc = x - sq.chunk[i];
        const int p = gc / sq.seg_chunks;
        if (p == 0) return;
        qe_idx = (long long)sq.chunk[i] * H + (long long)h * (sq.chunk[i + 1] - sq.chunk[i]) + gc;
        sb_idx = ((long long)sq.seg[i] + p) * H + h;
        row0 = (long long)sq.tok[i] + (long long)gc * C;
        L = min(C, (int)(sq.tok[i + 1] - row0));
    }
    pdl_wait();
    pdl_trigger();
    const long long tstride = (long long)H * DV;

    // every copy of the three tiles in flight at once
    {   // Qe rows (zero past the sequence end: a 0-byte source fills zeros)
        const __nv_bfloat16* src = Qe + (size_t)qe_idx * C * DK;
#pragma unroll
        for (int i = tid; i < C * DK / 8; i += THREADS) {
            const int r = i / (DK / 8), cc = i % (DK / 8);
            cp_async16(qs + r * LDA + cc * 8, src + (r < L ? i * 8 : 0), r < L ? 16u : 0u);
        }
    }
    {   // S* of the segment
        const __nv_bfloat16* src = Sb + (size_t)sb_idx * DV * DK;
#pragma unroll
        for (int i = tid; i < DV * DK / 8; i += THREADS) {
            const int r = i / (DK / 8), cc = i % (DK / 8);
            cp_async16(ss + r * LDA + cc * 8, src + i * 8, 16u);
        }
    }
    {   // the provisional outputs of the chunk (rows past the sequence end are never stored)
#pragma unroll
        for (int i = tid; i < C * DV / 8; i += THREADS) {
            const int r = i / (DV / 8), cc = i % (DV / 8);
            if (r < L) cp_async16(os + r * LDO + cc * 8, o + (row0 + r) * tstride + h * DV + cc * 8, 16u);
        }
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    // acc[m][n]: rows 16 m + (g, g + 8), columns n0 + 8 n + (2 t, 2 t + 1)
    float acc[4][NT][4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;
    const int n0 = warp * (DV / 8);
    const uint32_t qbase = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(ss));
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4][4], bb[NT][2];
#pragma unroll
        for (int m = 0; m < 4; ++m)     // A rows 16 m + (lane & 15), k-offset 8 (lane >> 4)
            ldsm_x4(qbase + (uint32_t)(((16 * m + (lane & 15)) * LDA + ks * 16 + (lane >> 4) * 8) * 2), a[m]);
#pragma unroll
        for (int n = 0; n < NT; ++n)    // B (S* rows = output columns) n0 + 8 n + (lane & 7), k-offset 8 ((lane >> 3) & 1)
            ldsm_x2(sbase + (uint32_t)(((n0 + 8 * n + (lane & 7)) * LDA + ks * 16 + ((lane >> 3) & 1) * 8) * 2),
                    bb[n]);
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int n = 0; n < NT; ++n) mma16816(acc[m][n], a[m], bb[n]);
    }
    // add into the staged outputs (each element is owned by one thread)
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = 16 * m + g + 8 * hr, col = n0 + 8 * n + 2 * t4;
                __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(os + r * LDO + col);
                const float2 cur = __bfloat1622float2(*op);
                *op = __floats2bfloat162_rn(cur.x + acc[m][n][2 * hr], cur.y + acc[m][n][2 * hr + 1]);
            }
    __syncthreads();
    for (int i = tid; i < C * DV / 8; i += THREADS) {
        const int r = i / (DV / 8), cc = i % (DV / 8);
        if (r < L)
            *reinterpret_cast<uint4*>(o + (row0 + r) * tstride + h * DV + cc * 8) =
                *reinterpret_cast<const uint4*>(os + r * LDO + cc * 8);
    }
}

}  // namespace pfcor
}  // namespace jet

namespace jet {
namespace pfcor {

// Dense layout, `ch` consecutive chunks of one segment per CTA (the host
// picks ch so that the grid is one wave of the SMs): S* is loaded once and
// the chunks' Qe and output tiles stream through NBUF buffers, NBUF - 1 chunks
// of copies in flight while one chunk's product is formed. Segments p0 =
// chunk0 / segc .. P-1; grid (groups of the segments, H, B) with
// ceil(segc / ch) groups per segment (a group past the sequence end returns
// at once).
constexpr int NBUF = 3;
constexpr int GTHREADS = 512;            // 16 warps: warp w owns output columns [w dv/16, (w+1) dv/16)
__host__ __device__ constexpr size_t smem_group_bytes(int dk, int dv) {
    return 2 * ((size_t)dv * lda(dk) + NBUF * (size_t)C * lda(dk) + NBUF * (size_t)C * ldo(dv));
}

template <int DK, int DV>
__global__ void __launch_bounds__(GTHREADS)
prefill_correct_group_kernel(const __nv_bfloat16* __restrict__ Qe, const __nv_bfloat16* __restrict__ Sb,
                             __nv_bfloat16* __restrict__ o, int Tn, int H, int nct, int chunk0, int segc, int P,
                             int ch) {
    static_assert(DK % 16 == 0 && DK <= 128 && DV % 64 == 0 && DV <= 256, "shapes");
    constexpr int LDA = lda(DK), LDO = ldo(DV);
    constexpr int NT = DV / 128;                 // n8 tiles per warp (DV / 16 columns)
    constexpr int KS = DK / 16;
    static_assert(NT >= 1, "dv >= 128");
    extern __shared__ __align__(16) uint8_t smem[];
    __nv_bfloat16* ss = reinterpret_cast<__nv_bfloat16*>(smem);          // [DV][LDA]
    __nv_bfloat16* qs0 = ss + DV * LDA;                                  // [NBUF][64][LDA]
    __nv_bfloat16* os0 = qs0 + NBUF * C * LDA;                           // [NBUF][64][LDO]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y, b = blockIdx.z;
    const int gps = (segc + ch - 1) / ch;                                // groups per segment
    const int p = chunk0 / segc + (int)blockIdx.x / gps;
    const int first = p * segc + ((int)blockIdx.x % gps) * ch;
    const int last = min(min(first + ch, (p + 1) * segc), nct);          // chunks [first, last)
    if (first >= last) return;
    const int n = last - first;
    pdl_wait();
    pdl_trigger();
    const long long tstride = (long long)H * DV;
    const long long row_b = (long long)b * Tn;

    auto issue_chunk = [&](int j) {      // Qe and output tiles of chunk first + j into buffer j % NBUF
        const int gc = first + j, L = min(C, Tn - gc * C);
        __nv_bfloat16* qs = qs0 + (j % NBUF) * C * LDA;
        __nv_bfloat16* os = os0 + (j % NBUF) * C * LDO;
        const __nv_bfloat16* src = Qe + (((long long)b * H + h) * nct + gc) * C * DK;
#pragma unroll
        for (int i = tid; i < C * DK / 8; i += GTHREADS) {
            const int r = i / (DK / 8), cc = i % (DK / 8);
            cp_async16(qs + r * LDA + cc * 8, src + (r < L ? i * 8 : 0), r < L ? 16u : 0u);
        }
        const long long row0 = row_b + (long long)gc * C;
#pragma unroll
        for (int i = tid; i < C * DV / 8; i += GTHREADS) {
            const int r = i / (DV / 8), cc = i % (DV / 8);
            if (r < L) cp_async16(os + r * LDO + cc * 8, o + (row0 + r) * tstride + h * DV + cc * 8, 16u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    {   // S* of the segment, in the first copy group with chunk 0
        const __nv_bfloat16* src = Sb + (((long long)b * P + p) * H + h) * DV * DK;
#pragma unroll
        for (int i = tid; i < DV * DK / 8; i += GTHREADS) {
            const int r = i / (DK / 8), cc = i % (DK / 8);
            cp_async16(ss + r * LDA + cc * 8, src + i * 8, 16u);
        }
    }
    for (int j = 0; j < NBUF - 1 && j < n; ++j) issue_chunk(j);

    const int n0 = warp * (DV / 16);
    const int g = lane >> 2, t4 = lane & 3;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(ss));
    for (int j = 0; j < n; ++j) {
        // chunk j's copies: the groups committed after it may stay in flight
        const int after = min(NBUF - 2, n - 1 - j);
        if (after >= 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
        else asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        // the buffer of chunk j - 1 is free (read out before the barrier): chunk j + NBUF - 1 into it
        if (j + NBUF - 1 < n) issue_chunk(j + NBUF - 1);
        __nv_bfloat16* qs = qs0 + (j % NBUF) * C * LDA;
        __nv_bfloat16* os = os0 + (j % NBUF) * C * LDO;
        const uint32_t qbase = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
        float acc[4][NT][4];
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int nn = 0; nn < NT; ++nn)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[m][nn][e] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t a[4][4], bb[NT][2];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                ldsm_x4(qbase + (uint32_t)(((16 * m + (lane & 15)) * LDA + ks * 16 + (lane >> 4) * 8) * 2), a[m]);
#pragma unroll
            for (int nn = 0; nn < NT; ++nn)
                ldsm_x2(sbase + (uint32_t)(((n0 + 8 * nn + (lane & 7)) * LDA + ks * 16 + ((lane >> 3) & 1) * 8) * 2),
                        bb[nn]);
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int nn = 0; nn < NT; ++nn) mma16816(acc[m][nn], a[m], bb[nn]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int nn = 0; nn < NT; ++nn)
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int r = 16 * m + g + 8 * hr, col = n0 + 8 * nn + 2 * t4;
                    __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(os + r * LDO + col);
                    const float2 cur = __bfloat1622float2(*op);
                    *op = __floats2bfloat162_rn(cur.x + acc[m][nn][2 * hr], cur.y + acc[m][nn][2 * hr + 1]);
                }
        __syncthreads();
        const int gc = first + j, L = min(C, Tn - gc * C);
        const long long row0 = row_b + (long long)gc * C;
        for (int i = tid; i < C * DV / 8; i += GTHREADS) {
            const int r = i / (DV / 8), cc = i % (DV / 8);
            if (r < L)
                *reinterpret_cast<uint4*>(o + (row0 + r) * tstride + h * DV + cc * 8) =
                    *reinterpret_cast<const uint4*>(os + r * LDO + cc * 8);
        }
    }
}

}  // namespace pfcor
}  // namespace jet
