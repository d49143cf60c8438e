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
// reads S0 while the last segment may be writing a final state that aliases it. Rows of S are independent, so each CTA owns 16 rows of one
// (sequence, head) and walks p sequentially; A_p is staged in shared memory.
#pragma once
#include "common.cuh"

namespace jet {

constexpr int SC_ROWS = 16;
constexpr int SC_THREADS = 256;

__host__ __device__ constexpr size_t sc_smem_bytes(int dk) {
    return sizeof(float) * ((size_t)dk * (dk + 1) + (size_t)SC_ROWS * (dk + 1));
}

// E [B][P-1][H][dv][dk], A [B][P-1][H][dk][dk], Sst [B][P][H][dv][dk]
__global__ void __launch_bounds__(SC_THREADS)
seg_combine_kernel(const float* __restrict__ E, const float* __restrict__ A, const float* S0,
                   float* __restrict__ Sst, int P, int H, int dv, int dk) {
    extern __shared__ float scm[];
    float* As = scm;                          // [dk][dk+1]
    float* Es = As + dk * (dk + 1);           // [16][dk+1]
    const int tid = threadIdx.x;
    const int r0 = blockIdx.x * SC_ROWS, h = blockIdx.y, b = blockIdx.z;
    const int ld = dk + 1;
    auto e_at = [&](int p) { return E + ((((long long)b * (P - 1) + p) * H + h) * dv + r0) * dk; };
    auto s_at = [&](int p) { return Sst + ((((long long)b * P + p) * H + h) * dv + r0) * dk; };
    // S_start(0) = S0, S_start(1) = E_0
    const float* s0 = S0 ? S0 + (((long long)b * H + h) * dv + r0) * dk : nullptr;
    for (int i = tid; i < SC_ROWS * dk; i += SC_THREADS) s_at(0)[i] = s0 ? s0[i] : 0.f;
    for (int i = tid; i < SC_ROWS * dk; i += SC_THREADS) {
        const int r = i / dk, j = i % dk;
        const float x = e_at(0)[(long long)r * dk + j];
        Es[r * ld + j] = x;
        s_at(1)[(long long)r * dk + j] = x;
    }
    for (int p = 1; p + 1 < P; ++p) {
        const float* Ap = A + ((((long long)b * (P - 1) + p) * H + h) * dk) * dk;
        __syncthreads();
        for (int i = tid; i < dk * dk; i += SC_THREADS) As[(i / dk) * ld + i % dk] = Ap[i];
        __syncthreads();
        float acc[SC_ROWS * 128 / SC_THREADS];           // outputs per thread (dk <= 128)
        const int nout = SC_ROWS * dk;
        int m = 0;
        for (int i = tid; i < nout; i += SC_THREADS, ++m) {
            const int r = i / dk, j = i % dk;
            float x = e_at(p)[(long long)r * dk + j];
            for (int q = 0; q < dk; ++q) x += Es[r * ld + q] * As[q * ld + j];
            acc[m] = x;
        }
        __syncthreads();
        m = 0;
        for (int i = tid; i < nout; i += SC_THREADS, ++m) {
            const int r = i / dk, j = i % dk;
            Es[r * ld + j] = acc[m];
            s_at(p + 1)[(long long)r * dk + j] = acc[m];
        }
    }
}

}  // namespace jet
