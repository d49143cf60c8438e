// K2 (CUDA-core form): chunked Gated DeltaNet prefill in float32 FFMA.
//
// Used for float32 inputs (where bf16 tensor-core operands would miss a 1e-4
// tolerance) and as the fallback shape for small heads. One CTA owns one
// (sequence, head, slice of DVS state rows) and walks the chunks of C = 64
// tokens in order, keeping its S slice [DVS][dk] in shared memory.
//
// Per chunk (gated delta rule, Jet-Nemotron paper section 2.3, rewritten in
// the chunked WY / UT-transform form; r, i index tokens of the chunk):
//   G_r = sum_{s<=r} g_s,  gam_r = exp(G_r)
//   A_ri = b_r exp(G_r - G_i) (k^_r . k^_i)   (i < r)
//   P_ri = exp(G_r - G_i) (q^_r . k^_i)       (i <= r)
//   (I + A) U = diag(b) V,  (I + A) W = diag(b gam) K^   (forward substitution)
//   Wt = U - W S^T
//   O  = diag(gam) Q^ S^T + P Wt
//   S <- gam_L S + Wt^T diag(exp(G_L - G_i)) K^
// Decay factors are always formed as exp(G_r - G_i) <= 1, never as a ratio
// of two exponentials, so deep cumulative gates underflow to 0 safely.
#pragma once
#include "common.cuh"

namespace jet {

constexpr int PS_THREADS = 256;
constexpr int PS_C = 64;
constexpr int PS_DVS = 32;      // state rows per CTA

__host__ __device__ constexpr int ps_smem_floats(int DK) {
    return 2 * PS_C * (DK + 1)          // Kc, Qc
         + PS_C * (DK + 1)              // Ws
         + PS_C * (PS_DVS + 1)          // Vs (b V -> U -> Wt)
         + 2 * PS_C * (PS_C + 1)        // A, P
         + PS_DVS * (DK + 1)            // S slice
         + 4 * PS_C;                    // G, gam, bet, dcy
}

template <typename T, int DK>
__global__ void __launch_bounds__(PS_THREADS)
gdn_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                        const float* __restrict__ g, const float* __restrict__ beta,
                        const float* S0, T* __restrict__ o, float* S_out,
                        int Tn, int H, int dv) {
    pdl_wait();
    pdl_trigger();
    constexpr int C = PS_C, DVS = PS_DVS, LD = DK + 1, LV = DVS + 1, LC = C + 1;
    extern __shared__ float sm[];
    float* Kc = sm;
    float* Qc = Kc + C * LD;
    float* Ws = Qc + C * LD;
    float* Vs = Ws + C * LD;
    float* A = Vs + C * LV;
    float* P = A + C * LC;
    float* Ss = P + C * LC;
    float* G = Ss + DVS * LD;
    float* gam = G + C;
    float* bet = gam + C;
    float* dcy = bet + C;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c0 = blockIdx.x * DVS, h = blockIdx.y, b = blockIdx.z;
    const long long bh = (long long)b * H + h;

    for (int i = tid; i < DVS * DK; i += PS_THREADS) {
        const int r = i / DK, j = i % DK;
        Ss[r * LD + j] = S0 ? S0[(bh * dv + c0 + r) * DK + j] : 0.f;
    }

    for (int t0 = 0; t0 < Tn; t0 += C) {
        const int L = min(C, Tn - t0);
        __syncthreads();
        // ---- load the chunk ----
        for (int i = tid; i < C * DK; i += PS_THREADS) {
            const int r = i / DK, j = i % DK;
            float kv = 0.f, qv = 0.f;
            if (r < L) {
                const long long off = (((long long)b * Tn + t0 + r) * H + h) * DK + j;
                kv = Elem<T>::ld(k + off);
                qv = Elem<T>::ld(q + off);
            }
            Kc[r * LD + j] = kv;
            Qc[r * LD + j] = qv;
        }
        for (int i = tid; i < C * DVS; i += PS_THREADS) {
            const int r = i / DVS, c = i % DVS;
            Vs[r * LV + c] = r < L ? Elem<T>::ld(v + (((long long)b * Tn + t0 + r) * H + h) * dv + c0 + c) : 0.f;
        }
        if (tid < C) {
            const long long off = ((long long)b * Tn + t0 + tid) * H + h;
            G[tid] = tid < L ? g[off] : 0.f;
            bet[tid] = tid < L ? beta[off] : 0.f;
        }
        __syncthreads();
        // ---- L2 norms (one warp per row), cumulative gate ----
        for (int r = warp; r < C; r += PS_THREADS / 32) {
            float sk = 0.f, sq = 0.f;
            for (int j = lane; j < DK; j += 32) {
                sk += Kc[r * LD + j] * Kc[r * LD + j];
                sq += Qc[r * LD + j] * Qc[r * LD + j];
            }
            sk = warp_sum(sk);
            sq = warp_sum(sq);
            const float ik = 1.0f / sqrtf(sk + 1e-6f), iq = 1.0f / sqrtf(sq + 1e-6f);
            for (int j = lane; j < DK; j += 32) {
                Kc[r * LD + j] *= ik;
                Qc[r * LD + j] *= iq;
            }
        }
        if (tid == 0) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += G[r]; G[r] = acc; }
        }
        __syncthreads();
        if (tid < C) {
            gam[tid] = expf(G[tid]);
            dcy[tid] = tid < L ? expf(G[L - 1] - G[tid]) : 0.f;
        }
        // ---- A, P ----
        for (int i = tid; i < C * C; i += PS_THREADS) {
            const int r = i / C, s = i % C;
            float kk = 0.f, qk = 0.f;
            if (s <= r) {
#pragma unroll 8
                for (int j = 0; j < DK; ++j) {
                    const float ks = Kc[s * LD + j];
                    kk += Kc[r * LD + j] * ks;
                    qk += Qc[r * LD + j] * ks;
                }
            }
            const float dec = s <= r ? expf(G[r] - G[s]) : 0.f;
            A[r * LC + s] = s < r ? bet[r] * dec * kk : 0.f;
            P[r * LC + s] = dec * qk;
        }
        __syncthreads();
        // right-hand sides: b V and b gam K^
        for (int i = tid; i < C * DVS; i += PS_THREADS) {
            const int r = i / DVS, c = i % DVS;
            Vs[r * LV + c] *= bet[r];
        }
        for (int i = tid; i < C * DK; i += PS_THREADS) {
            const int r = i / DK, j = i % DK;
            Ws[r * LD + j] = bet[r] * gam[r] * Kc[r * LD + j];
        }
        __syncthreads();
        // ---- forward substitution, one column per thread ----
        for (int col = tid; col < DVS + DK; col += PS_THREADS) {
            float* X = col < DVS ? (Vs + col) : (Ws + (col - DVS));
            const int ld = col < DVS ? LV : LD;
            for (int r = 1; r < L; ++r) {
                float x = X[r * ld];
                for (int i = 0; i < r; ++i) x -= A[r * LC + i] * X[i * ld];
                X[r * ld] = x;
            }
        }
        __syncthreads();
        // ---- Wt = U - W S^T ----
        for (int i = tid; i < C * DVS; i += PS_THREADS) {
            const int r = i / DVS, c = i % DVS;
            float ws = 0.f;
#pragma unroll 8
            for (int j = 0; j < DK; ++j) ws += Ws[r * LD + j] * Ss[c * LD + j];
            Vs[r * LV + c] -= ws;
        }
        __syncthreads();
        // ---- O = diag(gam) Q^ S^T + P Wt ----
        for (int i = tid; i < L * DVS; i += PS_THREADS) {
            const int r = i / DVS, c = i % DVS;
            float qs = 0.f;
#pragma unroll 8
            for (int j = 0; j < DK; ++j) qs += Qc[r * LD + j] * Ss[c * LD + j];
            float in = 0.f;
            for (int s = 0; s <= r; ++s) in += P[r * LC + s] * Vs[s * LV + c];
            Elem<T>::st(o + (((long long)b * Tn + t0 + r) * H + h) * dv + c0 + c, gam[r] * qs + in);
        }
        __syncthreads();
        // ---- S <- gam_L S + Wt^T diag(dcy) K^ ----
        const float gL = gam[L - 1];
        for (int i = tid; i < DVS * DK; i += PS_THREADS) {
            const int c = i / DK, j = i % DK;
            float s = gL * Ss[c * LD + j];
            for (int r = 0; r < L; ++r) s += Vs[r * LV + c] * dcy[r] * Kc[r * LD + j];
            Ss[c * LD + j] = s;
        }
    }
    __syncthreads();
    for (int i = tid; i < DVS * DK; i += PS_THREADS) {
        const int r = i / DK, j = i % DK;
        S_out[(bh * dv + c0 + r) * DK + j] = Ss[r * LD + j];
    }
}

}  // namespace jet
