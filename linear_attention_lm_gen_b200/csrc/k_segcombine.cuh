// Segment start states of the sequence-parallel prefill.
//
// The gated delta rule is affine in the state (Jet-Nemotron paper, section
// 2.3): over a segment, S_end = S_start A + B, with A (dk x dk) the product of
// the per-token transitions a_t (I - b_t k^_t k^_t^T) and B the end state
// reached from a zero start. Phase A of the prefill writes B_p (E below, with
// E_0 the true end state of segment 0) and A_p for p = 1 .. P-2; this kernel
// chains them:
//   S_start(1) = E_0,   S_start(p + 1) = S_start(p) A_p + E_p   (p = 1 .. P-2)
// in float32. It also copies S0 (or zeros) to S_start(0), so that phase C never
// reads S0 while the last segment may be writing a final state that aliases it.
//
// Rows of S are independent: a CTA owns 16 rows of one (sequence, head) and
// walks p sequentially. Thread (j, g) owns column j of rows 4g .. 4g+3, so its
// four accumulators are independent FMA chains; the 16 running rows sit in
// shared memory (read as broadcast float4), and A_p arrives by one bulk copy
// into a double buffer, the copy of A_{p+1} in flight while step p computes.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace jet {

constexpr int SC_ROWS = 16;      // state rows per CTA
constexpr int SC_RPT = 4;        // rows per thread
constexpr int SC_GROUPS = SC_ROWS / SC_RPT;

__host__ __device__ constexpr int sc_threads(int dk) { return SC_GROUPS * dk; }
__host__ __device__ constexpr size_t sc_smem_bytes(int dk) {
    return sizeof(float) * (2 * (size_t)dk * dk + (size_t)SC_ROWS * dk) + 2 * sizeof(uint64_t);
}

// E [B][P-1][H][dv][dk], A [B][P-1][H][dk][dk], Sst [B][P][H][dv][dk];
// grid (dv / 16, H, B), sc_threads(DK) threads, sc_smem_bytes(DK) shared.
template <int DK>
__global__ void __launch_bounds__(SC_GROUPS * DK)
seg_combine_kernel(const float* __restrict__ E, const float* __restrict__ A, const float* S0,
                   float* __restrict__ Sst, int P, int H, int dv) {
    extern __shared__ __align__(128) float scm[];
    float* As = scm;                                  // [2][DK][DK]
    float* Es = As + 2 * DK * DK;                     // [16][DK] running rows
    uint64_t* bar = reinterpret_cast<uint64_t*>(Es + SC_ROWS * DK);
    constexpr uint32_t ABYTES = DK * DK * sizeof(float);
    const int tid = threadIdx.x, j = tid % DK, grp = tid / DK;
    const int r0 = blockIdx.x * SC_ROWS, h = blockIdx.y, b = blockIdx.z;
    auto e_at = [&](int p) { return E + ((((long long)b * (P - 1) + p) * H + h) * dv + r0) * DK; };
    auto s_at = [&](int p) { return Sst + ((((long long)b * P + p) * H + h) * dv + r0) * DK; };
    auto a_at = [&](int p) { return A + (((long long)b * (P - 1) + p) * H + h) * DK * DK; };

    if (tid == 0) {
        sm100::mbar_init(&bar[0], 1);
        sm100::mbar_init(&bar[1], 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int p = 1; p <= 2 && p + 1 < P; ++p) {
            sm100::mbar_expect_tx(&bar[p - 1], ABYTES);
            sm100::bulk_load(As + (p - 1) * DK * DK, a_at(p), ABYTES, &bar[p - 1]);
        }
    // S_start(0) = S0 (or zeros), S_start(1) = E_0
    const float* s0 = S0 ? S0 + (((long long)b * H + h) * dv + r0) * DK : nullptr;
#pragma unroll
    for (int i = 0; i < SC_RPT; ++i) {
        const int r = grp * SC_RPT + i;
        s_at(0)[r * DK + j] = s0 ? s0[r * DK + j] : 0.f;
        const float x = e_at(0)[r * DK + j];
        Es[r * DK + j] = x;
        s_at(1)[r * DK + j] = x;
    }
    __syncthreads();

    for (int p = 1; p + 1 < P; ++p) {
        const int buf = (p - 1) & 1;
        const uint32_t parity = ((p - 1) >> 1) & 1;
        float acc[SC_RPT];
        const float* ep = e_at(p);
#pragma unroll
        for (int i = 0; i < SC_RPT; ++i) acc[i] = __ldcs(ep + (grp * SC_RPT + i) * DK + j);
        const bool ok = sm100::mbar_wait(&bar[buf], parity);
        if (!__syncthreads_and(ok)) return;           // timed out: error word already set
        const float* Ab = As + buf * DK * DK;
        const float* Eg = Es + grp * SC_RPT * DK;
#pragma unroll 4
        for (int q = 0; q < DK; q += 4) {
            const float a0 = Ab[q * DK + j], a1 = Ab[(q + 1) * DK + j];
            const float a2 = Ab[(q + 2) * DK + j], a3 = Ab[(q + 3) * DK + j];
#pragma unroll
            for (int i = 0; i < SC_RPT; ++i) {
                const float4 e = *reinterpret_cast<const float4*>(Eg + i * DK + q);
                acc[i] = fmaf(e.x, a0, fmaf(e.y, a1, fmaf(e.z, a2, fmaf(e.w, a3, acc[i]))));
            }
        }
        __syncthreads();                              // every read of Es and As[buf] done
        if (tid == 0 && p + 3 < P) {          // A_{p+2} is used by step p + 2 <= P - 2
            sm100::mbar_expect_tx(&bar[buf], ABYTES);
            sm100::bulk_load(As + buf * DK * DK, a_at(p + 2), ABYTES, &bar[buf]);
        }
        float* sp = s_at(p + 1);
#pragma unroll
        for (int i = 0; i < SC_RPT; ++i) {
            const int r = grp * SC_RPT + i;
            Es[r * DK + j] = acc[i];
            sp[r * DK + j] = acc[i];
        }
        __syncthreads();
    }
}

}  // namespace jet
