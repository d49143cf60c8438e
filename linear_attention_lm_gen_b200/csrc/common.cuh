// Shared device helpers of the JetBlock kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace jet {

// Per-device error word (0 = ok). Kernels OR status bits into it; the host
// reads and clears it in jet_device_error(). The library is one translation
// unit (jet_api.cu includes every kernel), so it is defined here.
enum : int { DEVERR_TIMEOUT = 1, DEVERR_DATA = 2 };
__device__ int g_dev_error;

__device__ __forceinline__ void flag_error(int bits) { atomicOr(&g_dev_error, bits); }

// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialization allowed, so it may be scheduled while the
// previous kernel on the stream is still running. pdl_wait() blocks until
// that kernel (and so all earlier work on the stream) has completed and its
// writes are visible; a kernel calls it before its first read of global
// memory, after its purely local set-up (barrier init, TMEM allocation,
// descriptor prefetch). pdl_trigger() lets the next kernel be scheduled early;
// the next kernel's own pdl_wait still waits for this one to finish. Both are
// no-ops when the launch had no such dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- element access for the two storage dtypes --------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
    static __device__ __forceinline__ float round(float v) { return v; }      // to the storage precision
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
    static __device__ __forceinline__ float round(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }
};

// 16-byte vector of a storage dtype <-> floats (8 bf16 or 4 f32 per 16 B)
template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    static __device__ __forceinline__ uint32_t pack2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // .x = a (low half)
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ uint4 pack(const float* f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
    }
};

// streaming (evict-first) 16-byte global load / store
__device__ __forceinline__ float4 ld_stream_f4(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream_f4(float4* p, const float4& v) { __stcs(p, v); }

// One output of the width-4 dynamic causal conv (Jet-Nemotron paper, section
// 2.4): v'_t = w0 v_t + w1 v_{t-1} + w2 v_{t-2} + w3 v_{t-3}, always evaluated
// in this order, so that every kernel that applies the conv (the generator /
// conv pass, the fused decode and the prefill chain) rounds identically.
__device__ __forceinline__ float conv4(const float4& w, float v0, float v1, float v2, float v3) {
    return fmaf(w.w, v3, fmaf(w.z, v2, fmaf(w.y, v1, w.x * v0)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace jet
