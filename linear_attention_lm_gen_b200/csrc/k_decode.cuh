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
// With CONV the kernel also applies the dynamic causal conv of the new token
// (Jet-Nemotron paper, section 2.4) to the raw v it reads: with the token's
// taps w (from the kernel generator) and the raw history v_{t-3..t-1},
//   v'_t = w0 v_t + w1 v_{t-1} + w2 v_{t-2} + w3 v_{t-3}
// rounded to the storage precision as the separate conv kernel stores it,
// and it writes the shifted history (v_{t-2}, v_{t-1}, v_t) for the next step.
//
// With `slots` (a state cache), sequence b's state and history are entry
// slots[b] of the pools S [n_slots][H][dv][dk] and hist [n_slots][3][H][dv];
// an index outside [0, n_slots) sets the device error word and the CTA
// touches nothing.
//
// Mapping: 4 lanes per row, each lane holding dk/16 float4 of the row in an
// interleaved pattern (lane p reads float4 p, p+4, ...): every load
// instruction of a warp covers 8 rows x 64 contiguous bytes. A thread owns
// two rows (r and r + 64), so a CTA of 256 threads covers 128 rows; grid
// (ceil(dv/128), H, B). The state loads are issued first, before the q / k
// normalisation prologue, so they are in flight while it runs; k^ and q^ are
// read from shared memory. State loads and stores use the streaming cache
// policy (the state is touched once per step).
#pragma once
#include "common.cuh"

namespace jet {

constexpr int DEC_THREADS = 256;
constexpr int DEC_ROWS = 128;    // rows of S per CTA (two per 4-lane group)

// history [B][3][H][dv], oldest first; taps [B][H][4]
struct DecConv {
    const float* taps;
    const void* hist_in;     // null: zero history
    void* hist_out;
};
// early != 0: the previous kernel on the stream is the same library call's
// generator / conv launch, which writes only the taps (CONV) or the values v
// (no CONV). Everything else the kernel reads was complete before that
// launch began, so the state rows and the token vectors are read before the
// wait for it, and only the taps / v after (the state stream of the first CTAs
// then overlaps the generator).

template <typename T, int NV, bool CONV = false>   // NV = dk / 16 float4 per lane
__global__ void __launch_bounds__(DEC_THREADS, NV <= 6 ? 3 : 2)   // 3 CTAs per SM where the registers allow
gdn_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ g, const float* __restrict__ beta,
                  float* __restrict__ S, T* __restrict__ o, int H, int dv, DecConv cv = {},
                  const int* __restrict__ slots = nullptr, int n_slots = 0, int early = 0) {
    constexpr int DK = NV * 16;
    __shared__ __align__(16) float sk[DK];
    __shared__ __align__(16) float sq[DK];
    __shared__ float red[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y, b = blockIdx.z;
    const long long bh = (long long)b * H + h;                // token inputs and outputs
    if (!early) pdl_wait();
    pdl_trigger();
    int sb = b;                                               // state / history entry
    if (slots) {
        sb = slots[b];
        if (sb < 0 || sb >= n_slots) {                        // whole CTA, before any access
            if (tid == 0) flag_error(DEVERR_DATA);
            return;
        }
    }
    const long long sbh = (long long)sb * H + h;
    const int part = lane & 3;
    const int row0 = blockIdx.x * DEC_ROWS + warp * 8 + (lane >> 2);
    const int row1 = row0 + 64;
    const bool ok0 = row0 < dv, ok1 = row1 < dv;

    // state rows first: the loads overlap the prologue below
    float4 s0[NV], s1[NV];
    {
        const float4* r0 = reinterpret_cast<const float4*>(S + (sbh * dv + (ok0 ? row0 : 0)) * DK);
        const float4* r1 = reinterpret_cast<const float4*>(S + (sbh * dv + (ok1 ? row1 : 0)) * DK);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            s0[i] = ok0 ? ld_stream_f4(r0 + part + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
            s1[i] = ok1 ? ld_stream_f4(r1 + part + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // the raw v (CONV) never comes from the previous launch; a conv's output may
    float vi0 = 0.f, vi1 = 0.f;
    auto load_v = [&]() {
        vi0 = ok0 ? Elem<T>::ld(v + bh * dv + row0) : 0.f;
        vi1 = ok1 ? Elem<T>::ld(v + bh * dv + row1) : 0.f;
    };
    if (CONV || !early) load_v();
    // conv inputs: the raw history of both rows (v_{t-3}, v_{t-2}, v_{t-1}), loaded
    // now and used only after the prologue below, so their latency overlaps it
    float hv0[3] = {0.f, 0.f, 0.f}, hv1[3] = {0.f, 0.f, 0.f};
    const long long hb = (long long)sb * 3 * H * dv + (long long)h * dv;  // history of (b, h), position 0
    const long long hs = (long long)H * dv;                               // slot stride
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (CONV) {
        if (!early) w = *reinterpret_cast<const float4*>(cv.taps + bh * 4);
        const T* hin = static_cast<const T*>(cv.hist_in);
        if (hin) {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                if (ok0) hv0[j] = Elem<T>::ld(hin + hb + j * hs + row0);
                if (ok1) hv1[j] = Elem<T>::ld(hin + hb + j * hs + row1);
            }
        }
    }
    const float a = expf(g[bh]);
    const float bt = beta[bh];

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

    // dot products of both rows with the raw k and q (normalised afterwards)
    float u0 = 0.f, p0 = 0.f, u1 = 0.f, p1 = 0.f;
    const float4* k4 = reinterpret_cast<const float4*>(sk);
    const float4* q4 = reinterpret_cast<const float4*>(sq);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const float4 kf = k4[part + 4 * i], qf = q4[part + 4 * i];
        u0 += s0[i].x * kf.x + s0[i].y * kf.y + s0[i].z * kf.z + s0[i].w * kf.w;
        p0 += s0[i].x * qf.x + s0[i].y * qf.y + s0[i].z * qf.z + s0[i].w * qf.w;
        u1 += s1[i].x * kf.x + s1[i].y * kf.y + s1[i].z * kf.z + s1[i].w * kf.w;
        p1 += s1[i].x * qf.x + s1[i].y * qf.y + s1[i].z * qf.z + s1[i].w * qf.w;
    }
#pragma unroll
    for (int m = 1; m <= 2; m <<= 1) {
        u0 += __shfl_xor_sync(0xffffffffu, u0, m);
        p0 += __shfl_xor_sync(0xffffffffu, p0, m);
        u1 += __shfl_xor_sync(0xffffffffu, u1, m);
        p1 += __shfl_xor_sync(0xffffffffu, p1, m);
    }
    u0 *= inv_k; u1 *= inv_k; p0 *= inv_q; p1 *= inv_q;
    if (early) {                                      // the previous launch's output from here on
        pdl_wait();
        if constexpr (CONV) w = *reinterpret_cast<const float4*>(cv.taps + bh * 4);
        else load_v();
    }
    if constexpr (CONV) {   // v' of both rows, and the shifted history
        T* hout = static_cast<T*>(cv.hist_out);
        auto conv_row = [&](int row, float raw, const float* hv) -> float {
            if (part == 0) {
                Elem<T>::st(hout + hb + row, hv[1]);
                Elem<T>::st(hout + hb + hs + row, hv[2]);
                Elem<T>::st(hout + hb + 2 * hs + row, raw);
            }
            return Elem<T>::round(conv4(w, raw, hv[2], hv[1], hv[0]));
        };
        if (ok0) vi0 = conv_row(row0, vi0, hv0);
        if (ok1) vi1 = conv_row(row1, vi1, hv1);
    }
    const float c0 = bt * vi0 - a * bt * u0;
    const float c1 = bt * vi1 - a * bt * u1;
    const float ck0 = c0 * inv_k, ck1 = c1 * inv_k;   // c k^ = (c / |k|) k
    if (ok0) {
        float4* w = reinterpret_cast<float4*>(S + (sbh * dv + row0) * DK);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const float4 kf = k4[part + 4 * i];
            st_stream_f4(w + part + 4 * i, make_float4(a * s0[i].x + ck0 * kf.x, a * s0[i].y + ck0 * kf.y,
                                                       a * s0[i].z + ck0 * kf.z, a * s0[i].w + ck0 * kf.w));
        }
        if (part == 0) Elem<T>::st(o + bh * dv + row0, a * p0 + c0 * kq);
    }
    if (ok1) {
        float4* w = reinterpret_cast<float4*>(S + (sbh * dv + row1) * DK);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const float4 kf = k4[part + 4 * i];
            st_stream_f4(w + part + 4 * i, make_float4(a * s1[i].x + ck1 * kf.x, a * s1[i].y + ck1 * kf.y,
                                                       a * s1[i].z + ck1 * kf.z, a * s1[i].w + ck1 * kf.w));
        }
        if (part == 0) Elem<T>::st(o + bh * dv + row1, a * p1 + c1 * kq);
    }
}

}  // namespace jet
