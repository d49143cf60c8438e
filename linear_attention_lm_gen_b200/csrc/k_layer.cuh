// The JetBlock layer around the mixer: the element-wise stages between the
// projections and the mixer, and between the mixer and the output projection.
//
// The Jet-Nemotron paper (section 2.4, new attention block design) takes the
// block's queries, keys, values and the generator input from the shared
// input x and applies the dynamic conv to V alone; it gives no form for the
// gates or the output. The layer here is the Gated DeltaNet layer without its
// short convolutions:
//   g = -softplus(x Wg), b = sigmoid(x Wb)             (per token and head)
//   u = o / sqrt(mean_dv(o^2) + eps) * gamma * SiLU(z) (per token and head; z = x Wz)
// with q, k, v, z and the logits of g and b from plain GEMMs, and y = u Wo.
#pragma once
#include "common.cuh"

namespace jet {
namespace layer {

constexpr float kRmsEps = 1e-6f;
constexpr int GATE_THREADS = 256;
constexpr int OUT_THREADS = 256;             // 8 warps, one (token, head) per warp

// gl, bl [n] float32 logits -> g = -softplus(gl), b = sigmoid(bl), in place.
__global__ void __launch_bounds__(GATE_THREADS)
gates_kernel(float* __restrict__ gl, float* __restrict__ bl, long long n) {
    pdl_wait();
    pdl_trigger();
    for (long long i = blockIdx.x * (long long)GATE_THREADS + threadIdx.x; i < n;
         i += (long long)gridDim.x * GATE_THREADS) {
        const float a = gl[i], c = bl[i];
        // softplus(a) = max(a, 0) + log1p(exp(-|a|)), exact in form for every a
        gl[i] = -(fmaxf(a, 0.f) + log1pf(expf(-fabsf(a))));
        bl[i] = 1.f / (1.f + expf(-c));
    }
}

// o, z [rows][dv] bf16 (rows = tokens x heads), gamma [dv] float32 ->
// u [rows][dv] bf16 (may be o itself: every element is read before the same
// thread writes it). One warp per row; lane l takes the 16-byte groups
// l, l + 32, ... of the row. dv % 8 == 0, dv <= 8 * 32 * GROUPS.
template <int GROUPS>
__global__ void __launch_bounds__(OUT_THREADS)
out_gate_kernel(const __nv_bfloat16* o, const __nv_bfloat16* __restrict__ z, const float* __restrict__ gamma,
                __nv_bfloat16* u, long long rows, int dv) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long long row = blockIdx.x * (long long)(OUT_THREADS / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int ng = dv / 8;
    using V = Vec16<__nv_bfloat16>;
    float fo[GROUPS][8], fz[GROUPS][8];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < GROUPS; ++j) {
        const int grp = lane + 32 * j;
        if (grp < ng) {
            V::unpack(*reinterpret_cast<const uint4*>(o + row * dv + grp * 8), fo[j]);
            V::unpack(*reinterpret_cast<const uint4*>(z + row * dv + grp * 8), fz[j]);
#pragma unroll
            for (int e = 0; e < 8; ++e) ss += fo[j][e] * fo[j][e];
        }
    }
    ss = warp_sum(ss);
    const float inv = 1.f / sqrtf(ss / (float)dv + kRmsEps);
#pragma unroll
    for (int j = 0; j < GROUPS; ++j) {
        const int grp = lane + 32 * j;
        if (grp < ng) {
            const float4 g0 = *reinterpret_cast<const float4*>(gamma + grp * 8);
            const float4 g1 = *reinterpret_cast<const float4*>(gamma + grp * 8 + 4);
            const float gm[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            float r[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float zz = fz[j][e];
                r[e] = fo[j][e] * inv * gm[e] * (zz / (1.f + expf(-zz)));
            }
            *reinterpret_cast<uint4*>(u + row * dv + grp * 8) = V::pack(r);
        }
    }
}

}  // namespace layer
}  // namespace jet
