// K3: one Gated DeltaNet decode step, fused and memory-bound.
//
// Per (sequence b, head h) the state S [dv][dk] float32 is read once and
// written once. Each row i of S is independent (Jet-Nemotron paper, section
// 2.3, gated delta rule restated per row):
//   u_i  = S_i . k^,   p_i = S_i . q^          (both from the same read of S_i)
//   c_i  = b v_i - a b u_i
//   S'_i = a S_i + c_i k^                        (written back in place)
//   o_i  = S'_i . q^ = a p_i + c_i (k^ . q^)
// so one pass over S gives both the update and the output.
//
// Mapping: 4 lanes per row, each lane holding dk/16 float4 of the row in an
// interleaved pattern (lane p reads float4 p, p+4, ...): every load
// instruction of a warp covers 8 rows x 64 contiguous bytes. 256 threads =
// 64 rows per CTA; grid (ceil(dv/64), H, B). State loads and stores use the
// streaming cache policy (the state is touched once per step).
#pragma once
#include "common.cuh"

namespace jet {

constexpr int DEC_THREADS = 256;
constexpr int DEC_ROWS = 64;    // rows of S per CTA

template <typename T, int NV>   // NV = dk / 16 float4 per lane
__global__ void __launch_bounds__(DEC_THREADS)
gdn_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta,
                  float* __restrict__ S, T* __restrict__ o, int H, int dv) {
    constexpr int DK = NV * 16;
    __shared__ float sk[DK], sq[DK];
    __shared__ float red[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y, b = blockIdx.z;
    const long long bh = (long long)b * H + h;

    for (int j = tid; j < DK; j += DEC_THREADS) {
        sk[j] = Elem<T>::ld(k + bh * DK + j);
        sq[j] = Elem<T>::ld(q + bh * DK + j);
    }
    __syncthreads();
    if (warp < 3) {
        float acc = 0.f;
        for (int j = lane; j < DK; j += 32)
            acc += warp == 0 ? sk[j] * sk[j] : (warp == 1 ? sq[j] * sq[j] : sk[j] * sq[j]);
        acc = warp_sum(acc);
        if (lane == 0) red[warp] = acc;
    }
    __syncthreads();
    const float inv_k = 1.0f / sqrtf(red[0] + 1e-6f);
    const float inv_q = 1.0f / sqrtf(red[1] + 1e-6f);
    const float kq = red[2] * inv_k * inv_q;          // k^ . q^
    const float a = expf(g[bh]);
    const float bt = beta[bh];

    const int part = lane & 3;
    const int row = blockIdx.x * DEC_ROWS + warp * 8 + (lane >> 2);
    if (row >= dv) return;

    float4 kf[NV], qf[NV], s[NV];
    const float4* Srow = reinterpret_cast<const float4*>(S + (bh * dv + row) * DK);
#pragma unroll
    for (int i = 0; i < NV; ++i) s[i] = ld_stream_f4(Srow + part + 4 * i);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int j = 4 * (part + 4 * i);
        kf[i] = make_float4(sk[j] * inv_k, sk[j + 1] * inv_k, sk[j + 2] * inv_k, sk[j + 3] * inv_k);
        qf[i] = make_float4(sq[j] * inv_q, sq[j + 1] * inv_q, sq[j + 2] * inv_q, sq[j + 3] * inv_q);
    }
    float u = 0.f, p = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        u += s[i].x * kf[i].x + s[i].y * kf[i].y + s[i].z * kf[i].z + s[i].w * kf[i].w;
        p += s[i].x * qf[i].x + s[i].y * qf[i].y + s[i].z * qf[i].z + s[i].w * qf[i].w;
    }
    u += __shfl_xor_sync(0xffffffffu, u, 1);
    u += __shfl_xor_sync(0xffffffffu, u, 2);
    p += __shfl_xor_sync(0xffffffffu, p, 1);
    p += __shfl_xor_sync(0xffffffffu, p, 2);

    const float vi = Elem<T>::ld(v + bh * dv + row);
    const float c = bt * vi - a * bt * u;
    float4* Sw = reinterpret_cast<float4*>(S + (bh * dv + row) * DK);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        float4 r;
        r.x = a * s[i].x + c * kf[i].x;
        r.y = a * s[i].y + c * kf[i].y;
        r.z = a * s[i].z + c * kf[i].z;
        r.w = a * s[i].w + c * kf[i].w;
        st_stream_f4(Sw + part + 4 * i, r);
    }
    if (part == 0) Elem<T>::st(o + bh * dv + row, a * p + c * kq);
}

}  // namespace jet
