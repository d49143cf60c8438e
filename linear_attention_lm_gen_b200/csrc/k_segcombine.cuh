// Segment start states of the sequence-parallel prefill.
//
// The gated delta rule is affine in the state (Jet-Nemotron paper, section
// 2.3): over a segment, S_end = S_start A + B, with A (dk x dk) the product of
// the per-token transitions a_t (I - b_t k^_t k^_t^T) and B the end state
// reached from a zero start. The segment passes write the end states E_p
// (E_0 is the true end state of segment 0, which starts from S0) and the
// transitions A_p (p >= 1); this kernel chains them:
//   S_start(1) = E_0,   S_start(p + 1) = S_start(p) A_p + E_p.
// Two layouts:
//   one pass (FINAL): E and A hold all P segments; the kernel writes
//     S_start(1 .. P-1) in bf16 (the operand of the output correction, Sb)
//     and the final state S_start(P) in float32 to S_out (which may alias S0:
//     segment 0 has read S0 before this kernel runs);
//   two passes: E and A hold segments 0 .. P-2 (the pass without outputs);
//     the kernel writes S_start(0 .. P-1), S_start(0) being a copy of S0 (or
//     zeros), so that the pass with outputs never reads S0 while the last
//     segment may be writing a final state that aliases it.
#pragma once
#include "common.cuh"
#include "k_prefill_common.cuh"
#include "sm100.cuh"

namespace jet {

constexpr int SC_ROWS = 16;      // state rows per CTA (the MMA's M)

__host__ __device__ constexpr int sc_threads(int dk) { return 4 * dk; }     // one warp per 8 columns
__host__ __device__ constexpr int sc_lde(int dk) { return dk + 4; }          // padded row stride of the rows
__host__ __device__ constexpr size_t sc_smem_bytes(int dk) {
    return sizeof(float) * (2 * (size_t)dk * pfws::trans_ld(dk) + 4 * (size_t)SC_ROWS * sc_lde(dk)) + 2 * sizeof(uint64_t);
}

namespace sc {
__device__ __forceinline__ uint32_t tf32_of(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// x = hi + lo, both representable in tf32
__device__ __forceinline__ void split(float x, uint32_t& hi, uint32_t& lo) {
    hi = tf32_of(x);
    lo = tf32_of(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
}  // namespace sc

// Where segment p's end state, transition and start state of sequence b live:
// sequence-major ([B][NE][H]...), the layout of the segment passes, or
// segment-major ([NE][B][H]...), the layout of per-rank ranges gathered from
// several GPUs. lda: row stride of a transition (trans_ld(dk) in the
// workspaces; dk for dense [dk][dk] transitions, copied row by row).
struct CombineLayout {
    int seg_major;
    int lda;
};

// E [B][NE][H][dv][dk], A [B][NE][H][dk][lda] (or segment-major), NE = P
// (FINAL) or P - 1; start states Sst [B][P][H][dv][dk] float32 (two passes)
// or Sb bf16 (FINAL, same layout as E); grid (dv / 16, H, B), sc_threads(DK)
// threads, sc_smem_bytes(DK) shared.
// Variable-length batches (FINAL, sq.nseq > 0): sequence b has segments
// sq.seg[b] .. sq.seg[b+1]-1 of E, A and Sb ([global segment][H]...); a
// sequence of one segment has nothing to combine (the pass wrote its final
// state).
template <int DK, bool FINAL>
__global__ void __launch_bounds__(4 * DK)
seg_combine_kernel(const float* __restrict__ E, const float* __restrict__ A, const float* S0,
                   float* __restrict__ Sst, __nv_bfloat16* __restrict__ Sb, float* S_out, int Pn, int H, int dv,
                   const CombineLayout lay, const __grid_constant__ pfws::SeqMap sq) {
    static_assert(DK % 8 == 0 && DK <= 128, "dk");
    const int P = sq.nseq > 0 ? sq.seg[blockIdx.z + 1] - sq.seg[blockIdx.z] : Pn;
    if (P < 2) return;                           // whole CTA, before any barrier
    const int NE = FINAL ? P : P - 1;            // segments with an end state / transition
    const int last = FINAL ? P - 1 : P - 2;      // the last step p computes S_start(p + 1)
    constexpr int LDE = sc_lde(DK);
    extern __shared__ __align__(128) float scm[];
    constexpr int LDAT = pfws::trans_ld(DK);
    float* As = scm;                                  // [2][DK][LDAT]
    // running rows S_start(p), split once into tf32 hi / lo parts: [2][hi, lo][16][LDE]
    uint32_t* Es = reinterpret_cast<uint32_t*>(As + 2 * DK * LDAT);
    uint64_t* bar = reinterpret_cast<uint64_t*>(Es + 4 * SC_ROWS * LDE);
    auto put_row = [&](int p, int r, int j, float x) {   // S_start(p)[r][j] into the running rows
        uint32_t* e = Es + (p & 1) * 2 * SC_ROWS * LDE + r * LDE + j;
        sc::split(x, e[0], e[SC_ROWS * LDE]);
    };
    constexpr uint32_t ABYTES = DK * LDAT * sizeof(float);
    const uint32_t a_bytes = lay.lda == LDAT ? ABYTES : DK * DK * (uint32_t)sizeof(float);   // per transition
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3, n0 = warp * 8;
    const int r0 = blockIdx.x * SC_ROWS, h = blockIdx.y, b = blockIdx.z, nb = gridDim.z;
    // (segment, sequence) -> index of the [H] block
    auto sb_idx = [&](int p, int n) {
        if (sq.nseq > 0) return (long long)sq.seg[b] + p;
        return lay.seg_major ? (long long)p * nb + b : (long long)b * n + p;
    };
    auto e_at = [&](int p) { return E + ((sb_idx(p, NE) * H + h) * dv + r0) * DK; };
    auto s_at = [&](int p) {                     // S_start(p) (two passes); the final state (FINAL)
        return (FINAL && p == P) ? S_out + (((long long)b * H + h) * dv + r0) * DK
                                 : Sst + ((((long long)b * P + p) * H + h) * dv + r0) * DK;
    };
    auto sb_at = [&](int p) { return Sb + ((sb_idx(p, NE) * H + h) * dv + r0) * DK; };
    auto a_at = [&](int p) { return A + (sb_idx(p, NE) * H + h) * DK * (long long)lay.lda; };
    // A_p into As[buf]: one bulk copy of the padded rows, or a copy per dense row
    auto load_a = [&](int p, int buf) {
        float* dst = As + buf * DK * LDAT;
        sm100::mbar_expect_tx(&bar[buf], a_bytes);
        if (lay.lda == LDAT) {
            sm100::bulk_load(dst, a_at(p), ABYTES, &bar[buf]);
        } else {
            for (int j = 0; j < DK; ++j)
                sm100::bulk_load(dst + j * LDAT, a_at(p) + (long long)j * lay.lda, DK * (uint32_t)sizeof(float),
                                 &bar[buf]);
        }
    };
    // this thread's accumulator entries: rows g and g+8, columns n0+2t and n0+2t+1
    auto load_frag = [&](const float* src, float* d) {
        const float2 x = *reinterpret_cast<const float2*>(src + g * DK + n0 + 2 * t);
        const float2 y = *reinterpret_cast<const float2*>(src + (g + 8) * DK + n0 + 2 * t);
        d[0] = x.x; d[1] = x.y; d[2] = y.x; d[3] = y.y;
    };

    if (tid == 0) {
        sm100::mbar_init(&bar[0], 1);
        sm100::mbar_init(&bar[1], 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();                                   // E, A and S0 are read from here on
    pdl_trigger();
    if (tid == 0)
        for (int p = 1; p <= 2 && p <= last; ++p) load_a(p, p - 1);
    // two passes: S_start(0) = S0 (or zeros); both: S_start(1) = E_0, also the running rows of step 1
    const float* s0 = (!FINAL && S0) ? S0 + (((long long)b * H + h) * dv + r0) * DK : nullptr;
    {   // every thread owns 4 of the 16 x DK entries; all loads first, then the stores
        constexpr int PER = SC_ROWS / 4;
        float xs[PER], x0[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + u * 4 * DK;
            xs[u] = e_at(0)[i];
            x0[u] = s0 ? s0[i] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + u * 4 * DK;
            if (!FINAL) {
                s_at(0)[i] = x0[u];
                s_at(1)[i] = xs[u];
            } else if (P > 1) {
                sb_at(1)[i] = __float2bfloat16_rn(xs[u]);
            }
            put_row(1, i / DK, i % DK, xs[u]);
        }
    }
    float e_next[4] = {0.f, 0.f, 0.f, 0.f};
    if (1 <= last) load_frag(e_at(1), e_next);
    __syncthreads();

    for (int p = 1; p <= last; ++p) {
        const int buf = (p - 1) & 1;
        const uint32_t parity = ((p - 1) >> 1) & 1;
        float d[4] = {e_next[0], e_next[1], e_next[2], e_next[3]};
        if (p + 1 <= last) load_frag(e_at(p + 1), e_next);  // in flight during this step
        const bool ok = sm100::mbar_wait(&bar[buf], parity);
        if (!__syncthreads_and(ok)) return;                  // timed out: error word already set
        const float* Ab = As + buf * DK * LDAT;
        const uint32_t* Eh = Es + (p & 1) * 2 * SC_ROWS * LDE;  // S_start(p) rows, hi parts
        const uint32_t* El = Eh + SC_ROWS * LDE;                 // lo parts
        // six independent accumulators (product kind x even / odd k-step) keep
        // the dependent MMA chains short
        float acc[2][3][4] = {};
#pragma unroll
        for (int k0 = 0; k0 < DK; k0 += 8) {
            const int par = (k0 >> 3) & 1;
            uint32_t ah[4], al[4], bh[2], bl[2];
            const int i0 = g * LDE + k0 + t, i1 = (g + 8) * LDE + k0 + t;
            ah[0] = Eh[i0]; ah[1] = Eh[i1]; ah[2] = Eh[i0 + 4]; ah[3] = Eh[i1 + 4];
            al[0] = El[i0]; al[1] = El[i1]; al[2] = El[i0 + 4]; al[3] = El[i1 + 4];
            sc::split(Ab[(k0 + t) * LDAT + n0 + g], bh[0], bl[0]);
            sc::split(Ab[(k0 + t + 4) * LDAT + n0 + g], bh[1], bl[1]);
            sc::mma(acc[par][0], al, bh);
            sc::mma(acc[par][1], ah, bl);
            sc::mma(acc[par][2], ah, bh);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
            d[e] += ((acc[0][0][e] + acc[1][0][e]) + (acc[0][1][e] + acc[1][1][e])) + (acc[0][2][e] + acc[1][2][e]);
        // S_start(p+1): to the next running-row buffer and to global
        put_row(p + 1, g, n0 + 2 * t, d[0]);
        put_row(p + 1, g, n0 + 2 * t + 1, d[1]);
        put_row(p + 1, g + 8, n0 + 2 * t, d[2]);
        put_row(p + 1, g + 8, n0 + 2 * t + 1, d[3]);
        if (FINAL && p + 1 < P) {                     // a start state: the correction's bf16 operand
            __nv_bfloat16* sp = sb_at(p + 1);
            *reinterpret_cast<__nv_bfloat162*>(sp + g * DK + n0 + 2 * t) = __floats2bfloat162_rn(d[0], d[1]);
            *reinterpret_cast<__nv_bfloat162*>(sp + (g + 8) * DK + n0 + 2 * t) = __floats2bfloat162_rn(d[2], d[3]);
        } else {                                      // float32: a start state (two passes) or the final state
            float* sp = s_at(p + 1);
            *reinterpret_cast<float2*>(sp + g * DK + n0 + 2 * t) = make_float2(d[0], d[1]);
            *reinterpret_cast<float2*>(sp + (g + 8) * DK + n0 + 2 * t) = make_float2(d[2], d[3]);
        }
        __syncthreads();                              // every read of As[buf] and of the old rows done
        if (tid == 0 && p + 2 <= last) load_a(p + 2, buf);   // A_{p+2} is used by step p + 2
    }
}

}  // namespace jet
