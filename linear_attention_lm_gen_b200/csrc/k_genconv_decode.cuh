// K1 for decode: the kernel generator and the dynamic causal conv of ONE new
// token per sequence (Jet-Nemotron paper, section 2.4), bf16.
//
// What it computes is the same as genconv_kernel with one token per sequence:
//   z = x W1 (d_model -> 32), h = SiLU(z), w = h W2 (32 -> H*4 taps),
//   v'[h,:] = w0 v_t + w1 v_{t-1} + w2 v_{t-2} + w3 v_{t-3}
// with v_{t-1..t-3} from the sequence's 3-token history, which is shifted by
// one token (the new history is v_{t-2}, v_{t-1}, v_t, copied bit for bit).
//
// The launch is short, so its time is a chain of latencies; the design keeps
// that chain to one round trip to memory:
//   * every global read of the CTA is issued first, together: the x rows and
//     W1 rows of the CTA's slice of d_model and its W2 columns by cp.async
//     into shared memory, and the v token and 3 history tokens of each of the
//     thread's conv items (up to MAXIT per thread) into registers;
//   * x . W1 on the tensor cores (bf16 mma.sync m16n8k16 with ldmatrix
//     operands, fp32 accumulate), the d_model reduction split across the G
//     CTAs of a thread-block cluster (one per head group) and the partial
//     sums added through distributed shared memory in rank order;
//   * the cluster barrier that keeps a CTA's partial sums alive until every
//     peer has read them is split: arrive after the reads, wait at the end,
//     so no CTA waits for it on the way to the conv.
// Conv items are one 16-byte channel group of one head of one token:
// consecutive threads take consecutive groups of a row (coalesced 128-bit
// loads and stores).
#pragma once
#include "common.cuh"
#include "k_genconv.cuh"

namespace jet {
namespace gcd {

constexpr int THREADS = 256;
constexpr int MAXIT = 4;                 // conv items per thread held in registers at once
constexpr int XPAD = 8;                  // bf16 padding of an x row (16 bytes: conflict-free ldmatrix)
constexpr int W1LD = GC_HID + 8;         // bf16 row stride of the W1 tile (80 bytes: conflict-free ldmatrix)
constexpr int ROWS = 16;                 // token rows of the x tile (one m16 tile; rows past TB are zero)

struct Layout {
    uint32_t xs, w1s, w2s, zpart, zc, hs, taps, bytes;
};
// kcols: d_model columns of the CTA's slice (a multiple of 16); cw: tap columns of the CTA
__host__ __device__ inline Layout layout(int kcols, int cw) {
    Layout L;
    uint32_t o = 0;
    L.xs = o;    o += (uint32_t)(ROWS * (kcols + XPAD) * 2);
    L.w1s = o;   o += (uint32_t)(kcols * W1LD * 2);
    L.w2s = o;   o += (uint32_t)((GC_HID * cw * 2 + 15) & ~15);
    L.zpart = o; o += 8u * ROWS * GC_HID * 4;
    L.zc = o;    o += (uint32_t)(ROWS * GC_HID * 4);
    L.hs = o;    o += (uint32_t)(ROWS * (GC_HID + 1) * 4);
    L.taps = o;  o += (uint32_t)(ROWS * cw * 4);
    L.bytes = o;
    return L;
}

__device__ __forceinline__ void cp_async(uint32_t dst, const void* src, uint32_t bytes, uint32_t src_bytes) {
    if (bytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Grid (ceil(B / TB), G), clusters of (1, G, 1): CTA (blk, g) owns tokens
// [blk TB, blk TB + TB) and heads [g hpc, g hpc + hpc), and reduces the
// d_model k-steps [g per, g per + per) of x . W1 for the cluster.
// slots (or null): sequence b's history is entry slots[b] of hist_in /
// hist_out, which may be the same pool (each element is read and rewritten by
// the one thread that owns it; the slots of one launch must differ). An index
// outside [0, n_slots) sets the device error word and the token's items are
// skipped. v == null: the taps only.
template <int TB>
__global__ void __launch_bounds__(THREADS, 2)
genconv_decode_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W1,
                      const __nv_bfloat16* __restrict__ W2, const __nv_bfloat16* __restrict__ v,
                      const __nv_bfloat16* hist_in, __nv_bfloat16* __restrict__ v_out, __nv_bfloat16* hist_out,
                      float* __restrict__ taps_out, int Bn, int D, int H, int dv, int hpc, int per,
                      const int* __restrict__ slots, int n_slots) {
    static_assert(TB == 8 || TB == 16, "token block");
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = (int)cluster_size(), g = (int)cluster_rank();
    const int h0 = blockIdx.y * hpc;
    const int nh = max(0, min(hpc, H - h0));
    const int CW = nh * GC_W, HW4 = H * GC_W;
    const int nks = D / 16;
    const int ks0 = min(nks, g * per), ks1 = min(nks, ks0 + per);
    const int kcols = per * 16;
    const int r0 = blockIdx.x * TB;
    const int nrows = min(TB, Bn - r0);
    const Layout L = layout(kcols, hpc * GC_W);
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const int ngrp = dv / 8;                       // 16-byte channel groups of a head row
    const int cols = nh * ngrp;
    const int items = v ? nrows * cols : 0;
    const long long rowstride = (long long)H * dv;

    pdl_wait();
    pdl_trigger();

    // ---- 1. every global read at once
    {   // x rows of the slice (rows past the block and columns past the slice read as zero)
        const int c8n = kcols / 8, kc8 = (ks1 - ks0) * 2;
        for (int i = tid; i < ROWS * c8n; i += THREADS) {
            const int r = i / c8n, c8 = i % c8n;
            const bool in = r < nrows && c8 < kc8;
            cp_async(sbase + L.xs + (uint32_t)(r * (kcols + XPAD) + c8 * 8) * 2,
                     in ? x + (long long)(r0 + r) * D + ks0 * 16 + c8 * 8 : x, 16, in ? 16 : 0);
        }
        // W1 rows of the slice
        const int kr_n = (ks1 - ks0) * 16;
        for (int i = tid; i < kcols * (GC_HID / 8); i += THREADS) {
            const int kr = i / (GC_HID / 8), c8 = i % (GC_HID / 8);
            const bool in = kr < kr_n;
            cp_async(sbase + L.w1s + (uint32_t)(kr * W1LD + c8 * 8) * 2,
                     in ? W1 + (long long)(ks0 * 16 + kr) * GC_HID + c8 * 8 : W1, 16, in ? 16 : 0);
        }
        // W2 columns of the CTA's heads: 4 bf16 (8 bytes) per (hidden unit, head)
        for (int i = tid; i < GC_HID * nh; i += THREADS) {
            const int r = i / nh, hl = i % nh;
            cp_async(sbase + L.w2s + (uint32_t)(r * CW + hl * GC_W) * 2, W2 + (long long)r * HW4 + (h0 + hl) * GC_W,
                     8, 8);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // conv items of the first batch: the token and its history, into registers
    uint4 cur[MAXIT], hw[MAXIT][3];
    int hq[MAXIT];
    auto item_load = [&](int it, uint4& c, uint4* w, int& hseq) {
        const int t = it / cols, col = it % cols;
        const int b = r0 + t;
        const long long coff = (long long)(h0 + col / ngrp) * dv + (long long)(col % ngrp) * 8;
        hseq = b;
        if (slots) {
            hseq = slots[b];
            if (hseq < 0 || hseq >= n_slots) { flag_error(DEVERR_DATA); hseq = -1; return; }
        }
        c = *reinterpret_cast<const uint4*>(v + (long long)b * rowstride + coff);
#pragma unroll
        for (int j = 0; j < 3; ++j)
            w[j] = hist_in ? *reinterpret_cast<const uint4*>(hist_in + ((long long)hseq * 3 + j) * rowstride + coff)
                           : make_uint4(0, 0, 0, 0);
    };
#pragma unroll
    for (int k = 0; k < MAXIT; ++k) {
        const int it = tid + k * THREADS;
        hq[k] = -1;
        if (it < items) item_load(it, cur[k], hw[k], hq[k]);
    }

    // ---- 2. this CTA's partial x . W1 over its slice (warp w takes k-steps w, w + 8, ...)
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    float* zpart = reinterpret_cast<float*>(smem + L.zpart);      // [8][ROWS][32]
    float* zc = reinterpret_cast<float*>(smem + L.zc);            // [ROWS][32]
    float* hs = reinterpret_cast<float*>(smem + L.hs);            // [ROWS][33]
    float* taps = reinterpret_cast<float*>(smem + L.taps);        // [ROWS][CW]
    const __nv_bfloat16* w2s = reinterpret_cast<const __nv_bfloat16*>(smem + L.w2s);   // [32][CW]
    {
        float acc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
        for (int kk = warp; kk < ks1 - ks0; kk += 8) {
            uint32_t a[4], b[4][2], r[4];
            ldsm_x4(sbase + L.xs + (uint32_t)(((lane & 15) * (kcols + XPAD) + kk * 16 + (lane >> 4) * 8) * 2), a);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                ldsm_x4_t(sbase + L.w1s +
                              (uint32_t)(((kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * W1LD + (2 * j + (lane >> 4)) * 8) * 2),
                          r);
                b[2 * j][0] = r[0]; b[2 * j][1] = r[1]; b[2 * j + 1][0] = r[2]; b[2 * j + 1][1] = r[3];
            }
#pragma unroll
            for (int n = 0; n < 4; ++n) mma_bf16_16816(acc[n], a, b[n]);
        }
        const int gq = lane >> 2, t4 = lane & 3;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            float* zp = zpart + (warp * ROWS + gq) * GC_HID + n * 8 + t4 * 2;
            zp[0] = acc[n][0];
            zp[1] = acc[n][1];
            zp[8 * GC_HID] = acc[n][2];
            zp[8 * GC_HID + 1] = acc[n][3];
        }
    }
    __syncthreads();
    for (int i = tid; i < TB * GC_HID; i += THREADS) {
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) z += zpart[w * ROWS * GC_HID + i];
        zc[i] = z;
    }
    // ---- 3. the cluster's partial sums, added in rank order by every CTA; SiLU
    cluster_sync_all();
    for (int i = tid; i < TB * GC_HID; i += THREADS) {
        float z = 0.f;
        for (int q = 0; q < G; ++q) z += ld_peer_f32(zc + i, (uint32_t)q);
        hs[(i / GC_HID) * (GC_HID + 1) + i % GC_HID] = z / (1.0f + expf(-z));
    }
    cluster_arrive();                                  // done with the peers' partial sums
    __syncthreads();

    // ---- 4. taps of this CTA's heads: h . W2 (hidden units in order)
    for (int i = tid; i < TB * CW; i += THREADS) {
        const int t = i / CW, c = i % CW;
        float acc = 0.f;
#pragma unroll 8
        for (int r = 0; r < GC_HID; ++r) acc += hs[t * (GC_HID + 1) + r] * __bfloat162float(w2s[r * CW + c]);
        taps[i] = acc;
        if (taps_out && t < nrows) taps_out[(long long)(r0 + t) * HW4 + h0 * GC_W + c] = acc;
    }
    __syncthreads();

    // ---- 5. the conv and the history shift
    auto item_store = [&](int it, const uint4& c, const uint4* w, int hseq) {
        if (hseq < 0) return;
        const int t = it / cols, col = it % cols;
        const int b = r0 + t, hl = col / ngrp;
        const long long coff = (long long)(h0 + hl) * dv + (long long)(col % ngrp) * 8;
        const float4 w4 = *reinterpret_cast<const float4*>(taps + t * CW + hl * GC_W);
        float fc[8], f1[8], f2[8], f3[8], out[8];
        Vec16<__nv_bfloat16>::unpack(c, fc);
        Vec16<__nv_bfloat16>::unpack(w[2], f1);            // v_{t-1}
        Vec16<__nv_bfloat16>::unpack(w[1], f2);            // v_{t-2}
        Vec16<__nv_bfloat16>::unpack(w[0], f3);            // v_{t-3}
#pragma unroll
        for (int e = 0; e < 8; ++e) out[e] = conv4(w4, fc[e], f1[e], f2[e], f3[e]);
        *reinterpret_cast<uint4*>(v_out + (long long)b * rowstride + coff) = Vec16<__nv_bfloat16>::pack(out);
        if (hist_out) {
            __nv_bfloat16* hp = hist_out + (long long)hseq * 3 * rowstride + coff;
            *reinterpret_cast<uint4*>(hp) = w[1];
            *reinterpret_cast<uint4*>(hp + rowstride) = w[2];
            *reinterpret_cast<uint4*>(hp + 2 * rowstride) = c;
        }
    };
#pragma unroll
    for (int k = 0; k < MAXIT; ++k) {
        const int it = tid + k * THREADS;
        if (it < items) item_store(it, cur[k], hw[k], hq[k]);
    }
    for (int base = MAXIT * THREADS; base < items; base += MAXIT * THREADS) {   // more items than registers
#pragma unroll
        for (int k = 0; k < MAXIT; ++k) {
            const int it = base + tid + k * THREADS;
            hq[k] = -1;
            if (it < items) item_load(it, cur[k], hw[k], hq[k]);
        }
#pragma unroll
        for (int k = 0; k < MAXIT; ++k) {
            const int it = base + tid + k * THREADS;
            if (it < items) item_store(it, cur[k], hw[k], hq[k]);
        }
    }
    cluster_wait();                                    // every peer has read this CTA's partial sums
}

}  // namespace gcd
}  // namespace jet
