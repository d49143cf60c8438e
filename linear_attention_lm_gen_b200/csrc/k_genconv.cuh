// K1: kernel generator fused with the dynamic causal conv on V.
//
// Jet-Nemotron paper, section 2.4: the generator shares the block input x,
// reduces it linearly (d_model -> 32), applies SiLU, and a final linear layer
// emits the conv taps (32 -> H*4). The taps of token t act on V only:
//   v'_t[h,:] = sum_{j=0..3} w_t[h,j] v_{t-j}[h,:]   (tap 0 = current token)
// with positions before token 0 taken from the history (or zero).
//
// One CTA owns TB consecutive tokens of the flattened [B*T] token axis and a
// group of heads; the G head-group CTAs of a token block form a thread-block
// cluster:
//   stage A  x[TB,D] . W1[D,32] split over the cluster: CTA g reduces the
//            g-th slice of D (bf16 tensor-core mma m16n8k16 with fp32
//            accumulate, the slice split again over the 8 warps; float32
//            inputs use FFMA), the partial sums meet in distributed shared
//            memory, and every CTA adds the G partials in the same order, so
//            x and W1 are read once per token block.
//   stage B  SiLU, then h[TB,32] . W2[32,H*4] in FFMA -> taps in shared memory
//            (and optionally to global).
//   stage C  conv: each work item is one 16-byte channel group of one head
//            over a run of tokens, holding a 3-token window in registers;
//            loads and stores are 128-bit and consecutive threads touch
//            consecutive 16-byte groups of a row (coalesced).
// The x.W1 product is ~6.5 flop per HBM byte of the kernel, so the tensor
// cores keep it in the shadow of the V stream.
#pragma once
#include "common.cuh"

namespace jet {

constexpr int GC_THREADS = 256;
constexpr int GC_HID = 32;      // generator hidden width
constexpr int GC_W = 4;         // conv width

// shared-memory layout (floats), TB tokens, CW = tap columns per CTA
__host__ __device__ constexpr int gc_smem_floats(int TB, int CW) {
    return 8 * TB * GC_HID      // partial sums of the 8 warps (bf16 path)
         + TB * GC_HID          // the CTA's partial sum (read by the cluster)
         + TB * (GC_HID + 1)    // hidden activations
         + GC_HID * CW          // W2 columns of the CTA's heads, as float
         + TB * CW;             // taps
}

__device__ __forceinline__ uint32_t ld_u32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint32_t pack_u16(uint16_t lo, uint16_t hi) { return (uint32_t)lo | ((uint32_t)hi << 16); }

// ---- thread-block cluster helpers (distributed shared memory)
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// the float at the same shared-memory offset in cluster CTA `rank`
__device__ __forceinline__ float ld_peer_f32(const float* p, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Stage A for bf16: z_part[warp][t][r] over the warp's share of the k-steps
// [ks0, ks1) (16 D-columns each).
template <int TB>
__device__ __forceinline__ void gen_stageA_bf16(const __nv_bfloat16* __restrict__ x,
                                                const __nv_bfloat16* __restrict__ W1,
                                                long long r0, long long N, int D, int ks0, int ks1, float* zpart) {
    constexpr int MT = TB / 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, t4 = lane & 3;
    const uint16_t* xs = reinterpret_cast<const uint16_t*>(x);
    const uint16_t* ws = reinterpret_cast<const uint16_t*>(W1);
    float acc[MT][4][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;

#pragma unroll 4
    for (int ks = ks0 + warp; ks < ks1; ks += 8) {
        const int k0 = ks * 16 + t4 * 2;
        uint32_t bfr[4][2];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int col = n * 8 + gid;
            bfr[n][0] = pack_u16(__ldg(ws + (long long)k0 * GC_HID + col), __ldg(ws + (long long)(k0 + 1) * GC_HID + col));
            bfr[n][1] = pack_u16(__ldg(ws + (long long)(k0 + 8) * GC_HID + col), __ldg(ws + (long long)(k0 + 9) * GC_HID + col));
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const long long ra = r0 + m * 16 + gid, rb = ra + 8;
            uint32_t afr[4];
            afr[0] = ra < N ? ld_u32(xs + ra * D + k0) : 0u;
            afr[1] = rb < N ? ld_u32(xs + rb * D + k0) : 0u;
            afr[2] = ra < N ? ld_u32(xs + ra * D + k0 + 8) : 0u;
            afr[3] = rb < N ? ld_u32(xs + rb * D + k0 + 8) : 0u;
#pragma unroll
            for (int n = 0; n < 4; ++n) mma_bf16_16816(acc[m][n], afr, bfr[n]);
        }
    }
    // accumulator fragment: rows gid / gid+8, cols t4*2, t4*2+1 of each n-tile
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            float* zp = zpart + (warp * TB + m * 16 + gid) * GC_HID + n * 8 + t4 * 2;
            zp[0] = acc[m][n][0];
            zp[1] = acc[m][n][1];
            zp[8 * GC_HID] = acc[m][n][2];
            zp[8 * GC_HID + 1] = acc[m][n][3];
        }
}

// Grid: x = blocks of TB tokens, y = G head groups of `hpc` heads, launched
// as clusters of (1, G, 1): the G CTAs of a token block split the x . W1
// reduction and share the result, and the taps and the conv are split across
// the head groups so that small token counts (decode: one token per
// sequence) still spread over many SMs.
// RUN = tokens per conv work item (8 keeps a sliding window in registers;
// 1 makes every token an independent item with its 4 loads in flight).
// slots (T = 1 and RUN = 1 only; the launcher refuses anything else, and the
// kernel ignores slots when RUN > 1): sequence b's history is entry slots[b] of hist_in /
// hist_out, which may then be the same pool: each history element is read
// and rewritten by the one thread that owns its item. An index outside
// [0, n_slots) sets the device error word and the item is skipped.
template <typename T, int TB, int RUN>
__global__ void __launch_bounds__(GC_THREADS, 2)
genconv_kernel(const T* __restrict__ x, const T* __restrict__ W1, const T* __restrict__ W2,
               const T* __restrict__ v, const T* hist_in, T* __restrict__ v_out,
               T* hist_out, float* __restrict__ conv_w_out,
               int Bn, int Tn, int D, int H, int dv, int hpc, const int* __restrict__ slots = nullptr,
               int n_slots = 0) {
    extern __shared__ float smem[];
    pdl_wait();
    pdl_trigger();
    const int HW4 = H * GC_W;
    const int h0 = blockIdx.y * hpc;
    const int nh = max(0, min(hpc, H - h0));
    const int CW = nh * GC_W;                     // tap columns of this CTA
    float* zpart = smem;                          // [8][TB][32]
    float* zc = zpart + 8 * TB * GC_HID;          // [TB][32] this CTA's partial sum
    float* hs = zc + TB * GC_HID;                 // [TB][33]
    float* w2s = hs + TB * (GC_HID + 1);          // [32][CW]
    float* taps = w2s + GC_HID * hpc * GC_W;      // [TB][CW]

    const int tid = threadIdx.x;
    const long long N = (long long)Bn * Tn;
    const long long r0 = (long long)blockIdx.x * TB;
    const int nrows = (int)((N - r0) < TB ? (N - r0) : TB);
    const int G = (int)cluster_size(), g = (int)cluster_rank();

    for (int i = tid; i < GC_HID * CW; i += GC_THREADS) {
        const int r = i / CW, c = i % CW;
        w2s[i] = Elem<T>::ld(W2 + (long long)r * HW4 + h0 * GC_W + c);
    }

    // ---- conv work items (stage C): one 16-byte channel group of one head
    // over a run of tokens. Their loads do not depend on the taps, so with one
    // token per item (decode) the first items' loads go out before stage A.
    using V16 = Vec16<T>;
    constexpr int VN = V16::N;                 // channels per 16-byte group
    constexpr int PF = RUN == 1 ? 2 : 0;       // items prefetched per thread
    const int ngrp = dv / VN;                  // groups per head row
    const int nruns = (nrows + RUN - 1) / RUN;
    const int cols = nh * ngrp;
    const int items = v ? cols * nruns : 0;
    const long long rowstride = (long long)H * dv;   // elements per token
    struct ItemGeo { long long rr0, coff; int hl, ta, tb, bseq, tpos0, hseq; };
    auto item_load = [&](int it, uint4* wraw, uint4* cur, ItemGeo& gi) {
        const int col = it % cols;
        const int run = it / cols;
        const int hl = col / ngrp, cg = col % ngrp;
        gi.hl = hl;
        gi.coff = (long long)(h0 + hl) * dv + (long long)cg * VN;
        gi.ta = run * RUN;
        gi.tb = min(nrows, gi.ta + RUN);
        gi.rr0 = r0 + gi.ta;
        gi.bseq = (int)(gi.rr0 / Tn);               // one division per item; then stepped
        gi.tpos0 = (int)(gi.rr0 - (long long)gi.bseq * Tn);
        gi.hseq = gi.bseq;                          // history entry of the sequence
        if (RUN == 1 && slots) {                    // slots only with one token per item (never crosses a sequence)
            gi.hseq = slots[gi.bseq];
            if (gi.hseq < 0 || gi.hseq >= n_slots) {
                flag_error(DEVERR_DATA);
                gi.tb = gi.ta;                      // nothing to do
                gi.hseq = -1;
            }
        }
        // window: wraw[0] = v_{t-1}, wraw[1] = v_{t-2}, wraw[2] = v_{t-3}
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int tau = gi.tpos0 - 1 - j;
            wraw[j] = make_uint4(0, 0, 0, 0);
            if (tau >= 0) wraw[j] = *reinterpret_cast<const uint4*>(v + (gi.rr0 - 1 - j) * rowstride + gi.coff);
            else if (hist_in && gi.hseq >= 0)
                wraw[j] = *reinterpret_cast<const uint4*>(hist_in + ((long long)gi.hseq * 3 + (3 + tau)) * rowstride + gi.coff);
        }
#pragma unroll
        for (int i = 0; i < RUN; ++i)
            if (gi.ta + i < gi.tb) cur[i] = *reinterpret_cast<const uint4*>(v + (gi.rr0 + i) * rowstride + gi.coff);
    };
    auto item_compute = [&](const uint4* wraw, const uint4* cur, const ItemGeo& gi) {
        const long long coff = gi.coff;
        int bseq = gi.bseq;
        float win[3][VN];
#pragma unroll
        for (int j = 0; j < 3; ++j) V16::unpack(wraw[j], win[j]);
        int tpos = gi.tpos0;
#pragma unroll
        for (int i = 0; i < RUN; ++i) {
            if (gi.ta + i >= gi.tb) break;
            const long long rr = gi.rr0 + i;
            if (RUN > 1 && i > 0 && tpos == Tn) {      // a new sequence starts inside the run
                tpos = 0;
                ++bseq;
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    uint4 u = make_uint4(0, 0, 0, 0);
                    if (hist_in) u = *reinterpret_cast<const uint4*>(hist_in + ((long long)bseq * 3 + (2 - j)) * rowstride + coff);
                    V16::unpack(u, win[j]);
                }
            }
            float cv[VN];
            V16::unpack(cur[i], cv);
            const float4 w4 = *reinterpret_cast<const float4*>(taps + (gi.ta + i) * CW + gi.hl * GC_W);
            float out[VN];
#pragma unroll
            for (int e = 0; e < VN; ++e)
                out[e] = conv4(w4, cv[e], win[0][e], win[1][e], win[2][e]);
            *reinterpret_cast<uint4*>(v_out + rr * rowstride + coff) = V16::pack(out);
#pragma unroll
            for (int e = 0; e < VN; ++e) { win[2][e] = win[1][e]; win[1][e] = win[0][e]; win[0][e] = cv[e]; }
            if (hist_out && tpos == Tn - 1) {
                const long long hq = (RUN == 1 && slots) ? gi.hseq : bseq;
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    *reinterpret_cast<uint4*>(hist_out + (hq * 3 + (2 - j)) * rowstride + coff) = V16::pack(win[j]);
            }
            ++tpos;
        }
    };
    uint4 pw[PF > 0 ? PF : 1][3], pc[PF > 0 ? PF : 1][RUN];
    ItemGeo pg[PF > 0 ? PF : 1];
#pragma unroll
    for (int q = 0; q < PF; ++q)
        if (tid + q * GC_THREADS < items) item_load(tid + q * GC_THREADS, pw[q], pc[q], pg[q]);

    // ---- stage A: this CTA's slice of z = x . W1 ----
    const int nks = D / 16, per = (nks + G - 1) / G;
    const int ks0 = min(nks, g * per), ks1 = min(nks, ks0 + per);
    if constexpr (sizeof(T) == 2) {
        gen_stageA_bf16<TB>(reinterpret_cast<const __nv_bfloat16*>(x),
                            reinterpret_cast<const __nv_bfloat16*>(W1), r0, N, D, ks0, ks1, zpart);
        __syncthreads();
        for (int i = tid; i < TB * GC_HID; i += GC_THREADS) {
            const int t = i / GC_HID, r = i % GC_HID;
            float z = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) z += zpart[(w * TB + t) * GC_HID + r];
            zc[i] = z;
        }
    } else {
        // float32: thread (t, 4 hidden units) in FFMA over the slice
        for (int i = tid; i < TB * (GC_HID / 4); i += GC_THREADS) {
            const int t = i / (GC_HID / 4), r4 = (i % (GC_HID / 4)) * 4;
            float z[4] = {0.f, 0.f, 0.f, 0.f};
            if (t < nrows) {
                const T* xr = x + (r0 + t) * D;
                for (int d = ks0 * 16; d < ks1 * 16; ++d) {
                    const float xv = Elem<T>::ld(xr + d);
#pragma unroll
                    for (int e = 0; e < 4; ++e) z[e] += xv * Elem<T>::ld(W1 + (long long)d * GC_HID + r4 + e);
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) zc[t * GC_HID + r4 + e] = z[e];
        }
    }
    // ---- the cluster's partial sums, added in rank order by every CTA; SiLU ----
    cluster_sync_all();
    for (int i = tid; i < TB * GC_HID; i += GC_THREADS) {
        const int t = i / GC_HID, r = i % GC_HID;
        float z = 0.f;
        for (int q = 0; q < G; ++q) z += ld_peer_f32(zc + i, (uint32_t)q);
        hs[t * (GC_HID + 1) + r] = z / (1.0f + expf(-z));
    }
    cluster_sync_all();                           // peers have read this CTA's partial
    __syncthreads();

    // ---- stage B: taps of this CTA's heads = h . W2 ----
    for (int i = tid; i < TB * CW; i += GC_THREADS) {
        const int t = i / CW, c = i % CW;
        float acc = 0.f;
#pragma unroll 8
        for (int r = 0; r < GC_HID; ++r) acc += hs[t * (GC_HID + 1) + r] * w2s[r * CW + c];
        taps[i] = acc;
        if (conv_w_out && t < nrows) conv_w_out[(r0 + t) * HW4 + h0 * GC_W + c] = acc;
    }
    if (v == nullptr) return;
    __syncthreads();

    // ---- stage C: causal conv over V ----
#pragma unroll
    for (int q = 0; q < PF; ++q)
        if (tid + q * GC_THREADS < items) item_compute(pw[q], pc[q], pg[q]);
    for (int it = tid + PF * GC_THREADS; it < items; it += GC_THREADS) {
        ItemGeo gg;
        uint4 wraw[3], cur[RUN];
        item_load(it, wraw, cur, gg);
        item_compute(wraw, cur, gg);
    }
}

}  // namespace jet
