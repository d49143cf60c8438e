// K1g: the kernel generator alone, for prompts (Jet-Nemotron paper, section
// 2.4: a linear reduction of the block input to 32, SiLU, and a linear layer
// that emits the H x 4 conv taps of every token):
//   taps[t][h*4 + j] = (SiLU(x_t W1) W2)[h*4 + j]      bf16 x, W1, W2; float32 out
//
// One CTA = GT = 32 consecutive tokens of the flattened [B*T] token axis.
// x[GT][D] and W1[D][32] stream through shared memory in slices of KC = 128
// columns of D (cp.async, NST - 1 slices in flight; four buffers, 75 KB, leave
// room on the SM for two CTAs of the chunk preparation that follows, which
// starts before this kernel ends); CTA b starts at slice
// b mod (slices), so the CTAs do not all ask for the same W1 lines at once. In every slice warp w takes
// k-step w (16 columns) of the whole 32 x 32 product: 2 x 4 bf16
// m16n8k16 tensor-core MMAs with float32 accumulation, operands by ldmatrix
// (W1 transposed on the fly). The 8 partial products meet in shared memory
// (added in warp order), then SiLU and h W2 in FFMA.
// The x . W1 product is ~21 flop per byte of x, so the kernel streams x at
// the memory system's pace when every SM holds a CTA.
#pragma once
#include "common.cuh"

namespace jet {
namespace kgen {

constexpr int THREADS = 256;
constexpr int GT = 32;                  // tokens per CTA
constexpr int HID = 32;                 // generator hidden width
constexpr int KC = 128;                 // columns of D per slice
constexpr int NST = 4;                  // slice buffers (NST - 1 in flight)
constexpr int XLD = KC * 2 + 16;        // x slice row stride in bytes (16-byte pad: conflict-free ldmatrix)
constexpr int WLD = HID * 2 + 16;       // W1 slice row stride in bytes
constexpr int XS_BYTES = GT * XLD;      // 8704
constexpr int WS_BYTES = KC * WLD;      // 10240
constexpr int ST_BYTES = XS_BYTES + WS_BYTES;
constexpr int PART_BYTES = 8 * GT * HID * 4;   // partial sums of the 8 warps (aliases the slices)
static_assert(NST * ST_BYTES >= PART_BYTES, "partials fit over the slice buffers");

constexpr int HLD = HID + 4;            // hidden-activation row stride (floats; 16-byte rows, rows on distinct banks)

__host__ __device__ constexpr int smem_bytes(int /*HW4*/) { return NST * ST_BYTES + GT * HLD * 4; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x [N][D], W1 [D][32], W2 [32][HW4] bf16; taps [N][HW4] float32. D % 16 == 0, HW4 <= 256.
__global__ void __launch_bounds__(THREADS)
gen_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W1,
           const __nv_bfloat16* __restrict__ W2, float* __restrict__ taps, long long N, int D, int HW4) {
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_wait();
    pdl_trigger();
    float* hs = reinterpret_cast<float*>(smem + NST * ST_BYTES);          // [GT][HLD] hidden activations
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long r0 = (long long)blockIdx.x * GT;
    const int nsl = (D + KC - 1) / KC;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));

    // this thread's copies of a slice: x rows xr, xr + 16 (16 bytes at column 8 * xc of the slice),
    // W1 rows wr, wr + 64 (16 bytes at column 8 * wc)
    const int xr = tid >> 4, xc = tid & 15, wr = tid >> 2, wc = tid & 3;
    const bool xok0 = r0 + xr < N, xok1 = r0 + xr + 16 < N;
    const __nv_bfloat16* xs0 = x + (xok0 ? (r0 + xr) * D : 0) + xc * 8;
    const __nv_bfloat16* xs1 = x + (xok1 ? (r0 + xr + 16) * D : 0) + xc * 8;
    const __nv_bfloat16* ws0 = W1 + (long long)wr * HID + wc * 8;
    const uint32_t xd = (uint32_t)(xr * XLD + xc * 16), wd = (uint32_t)(XS_BYTES + wr * WLD + wc * 16);
    // slices are read starting at slice (b mod nsl), so the CTAs spread their W1 requests
    int knext = (int)(blockIdx.x % (unsigned)nsl) * KC;         // column of the next slice to issue
    int kcur = knext;                                            // column of the next slice to compute
    auto issue = [&](int stage) {
        const uint32_t st = sbase + (uint32_t)stage * ST_BYTES;
        const int k0 = knext;
        knext = k0 + KC >= nsl * KC ? 0 : k0 + KC;
        // a copy of 0 bytes (zero fill) still gets an address inside the tensor
        const bool xin = k0 + xc * 8 < D;
        cp_async16(st + xd, xin && xok0 ? xs0 + k0 : x, xin && xok0 ? 16u : 0u);
        cp_async16(st + xd + 16 * XLD, xin && xok1 ? xs1 + k0 : x, xin && xok1 ? 16u : 0u);
        const bool w0 = k0 + wr < D, w1 = k0 + wr + 64 < D;
        cp_async16(st + wd, w0 ? ws0 + (long long)k0 * HID : W1, w0 ? 16u : 0u);
        cp_async16(st + wd + 64 * WLD, w1 ? ws0 + (long long)(k0 + 64) * HID : W1, w1 ? 16u : 0u);
    };
#pragma unroll
    for (int s = 0; s < NST - 1; ++s) {
        if (s < nsl) issue(s);
        cp_async_commit();
    }
    // this thread's W2 column for the last stage (bf16 pairs), loaded while the slices stream in
    const int ng = THREADS / HW4;                  // token groups of the h W2 stage
    const int col = tid % HW4, tg = tid / HW4;
    uint32_t w2p[HID / 2];
#pragma unroll
    for (int r = 0; r < HID; r += 2) {
        const uint16_t lo = tg < ng ? reinterpret_cast<const uint16_t*>(W2)[(long long)r * HW4 + col] : 0;
        const uint16_t hi = tg < ng ? reinterpret_cast<const uint16_t*>(W2)[(long long)(r + 1) * HW4 + col] : 0;
        w2p[r / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
    }

    float acc[2][4][4];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;

    // ldmatrix row addresses: A (x, row-major, non-transposed) rows (lane & 15), k-offset 8 (lane >> 4);
    // B (W1 [k][n], transposed) k-rows (lane & 15) of n-tile pair (lane >> 4)
    const uint32_t a_off = (uint32_t)((lane & 15) * XLD + (warp * 16 + (lane >> 4) * 8) * 2);
    const uint32_t b_off = (uint32_t)(XS_BYTES + (warp * 16 + (lane & 15)) * WLD + (lane >> 4) * 16);
    int stage = 0;
    for (int s = 0; s < nsl; ++s) {
        cp_async_wait<NST - 2>();                  // slice s has landed (this thread's copies)
        __syncthreads();                           // ... everyone's; stage (s-1) % NST is free
        if (s + NST - 1 < nsl) issue(stage == 0 ? NST - 1 : stage - 1);
        cp_async_commit();
        const uint32_t st = sbase + (uint32_t)stage * ST_BYTES;
        if (kcur + warp * 16 < D) {                // this warp's k-step exists
            uint32_t a[2][4], b[2][4];
            ldsm_x4(st + a_off, a[0]);
            ldsm_x4(st + a_off + 16 * XLD, a[1]);
            ldsm_x4_t(st + b_off, b[0]);                 // n-tiles 0, 1
            ldsm_x4_t(st + b_off + 32, b[1]);            // n-tiles 2, 3
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n)
                    mma16816(acc[m][n], a[m], b[n >> 1][(n & 1) * 2], b[n >> 1][(n & 1) * 2 + 1]);
        }
        kcur = kcur + KC >= nsl * KC ? 0 : kcur + KC;
        stage = stage + 1 == NST ? 0 : stage + 1;
    }
    cp_async_wait<0>();
    __syncthreads();                               // slices consumed: reuse them for the partial sums

    float* part = reinterpret_cast<float*>(smem);  // [8][GT][32]
    {
        const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                float* p = part + (warp * GT + m * 16 + g) * HID + n * 8 + t4 * 2;
                p[0] = acc[m][n][0];
                p[1] = acc[m][n][1];
                p[8 * HID] = acc[m][n][2];
                p[8 * HID + 1] = acc[m][n][3];
            }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < GT * HID / THREADS; ++q) {   // z = sum of the 8 partials (warp order), SiLU
        const int i = tid + q * THREADS, t = i / HID, r = i % HID;
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) z += part[w * GT * HID + i];
        hs[t * HLD + r] = z / (1.0f + expf(-z));
    }
    __syncthreads();
    if (tg >= ng) return;
    float w2[HID];
#pragma unroll
    for (int r = 0; r < HID / 2; ++r) {
        w2[2 * r] = __uint_as_float(w2p[r] << 16);
        w2[2 * r + 1] = __uint_as_float(w2p[r] & 0xffff0000u);
    }
    const int nrows = (int)(N - r0 < GT ? N - r0 : GT);
    for (int t = tg; t < nrows; t += ng) {
        const float4* hr = reinterpret_cast<const float4*>(hs + t * HLD);
        float a = 0.f;
#pragma unroll
        for (int r4 = 0; r4 < HID / 4; ++r4) {
            const float4 hv = hr[r4];
            a = fmaf(hv.x, w2[4 * r4], a);
            a = fmaf(hv.y, w2[4 * r4 + 1], a);
            a = fmaf(hv.z, w2[4 * r4 + 2], a);
            a = fmaf(hv.w, w2[4 * r4 + 3], a);
        }
        taps[(r0 + t) * HW4 + col] = a;
    }
}


// Long prompts: one CTA = WGT = 128 tokens, and warp w owns token rows
// [16 w, 16 w + 16) through every k-step of every slice, so W1 is read once
// per 128 tokens instead of once per 32 (at T = 262144 that is 201 MB of W1
// reads instead of 805, as much as the x stream itself) and no partial sums
// meet across warps. Slices of WKC = 64 columns, WNST - 1 in flight; 89 KB
// of shared memory, two CTAs per SM.
constexpr int WGT = 128, WKC = 64, WNST = 3;
constexpr int WXLD = WKC * 2 + 16;              // x row stride in a slice (bytes)
constexpr int WXS_BYTES = WGT * WXLD;           // 18432
constexpr int WST_BYTES = WXS_BYTES + WKC * WLD;   // + the W1 rows of the slice
__host__ __device__ constexpr int wide_smem_bytes() { return WNST * WST_BYTES + WGT * HLD * 4; }

__global__ void __launch_bounds__(THREADS, 2)
gen_wide_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W1,
                const __nv_bfloat16* __restrict__ W2, float* __restrict__ taps, long long N, int D, int HW4) {
    extern __shared__ __align__(16) uint8_t smem[];
    pdl_wait();
    pdl_trigger();
    float* hs = reinterpret_cast<float*>(smem + WNST * WST_BYTES);        // [WGT][HLD] hidden activations
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long r0 = (long long)blockIdx.x * WGT;
    const int nsl = (D + WKC - 1) / WKC;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    // this thread's copies of a slice: x rows xr + 32 j (16 bytes at column 8 xc), W1 row wr (column 8 wc)
    const int xr = tid >> 3, xc = tid & 7, wr = tid >> 2, wc = tid & 3;
    int knext = (int)(blockIdx.x % (unsigned)nsl) * WKC;
    int kcur = knext;
    auto issue = [&](int stage) {
        const uint32_t st = sbase + (uint32_t)stage * WST_BYTES;
        const int k0 = knext;
        knext = k0 + WKC >= nsl * WKC ? 0 : k0 + WKC;
        const bool xin = k0 + xc * 8 < D;
#pragma unroll
        for (int j = 0; j < WGT / 32; ++j) {
            const long long row = r0 + xr + 32 * j;
            const bool ok = xin && row < N;
            cp_async16(st + (uint32_t)((xr + 32 * j) * WXLD + xc * 16), ok ? x + row * D + k0 + xc * 8 : x,
                       ok ? 16u : 0u);
        }
        const bool win = k0 + wr < D;
        cp_async16(st + (uint32_t)(WXS_BYTES + wr * WLD + wc * 16),
                   win ? W1 + (long long)(k0 + wr) * HID + wc * 8 : W1, win ? 16u : 0u);
    };
#pragma unroll
    for (int s = 0; s < WNST - 1; ++s) {
        if (s < nsl) issue(s);
        cp_async_commit();
    }
    const int ng = THREADS / HW4;
    const int col = tid % HW4, tg = tid / HW4;
    uint32_t w2p[HID / 2];
#pragma unroll
    for (int r = 0; r < HID; r += 2) {
        const uint16_t lo = tg < ng ? reinterpret_cast<const uint16_t*>(W2)[(long long)r * HW4 + col] : 0;
        const uint16_t hi = tg < ng ? reinterpret_cast<const uint16_t*>(W2)[(long long)(r + 1) * HW4 + col] : 0;
        w2p[r / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    float acc[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
    // ldmatrix rows: A (x) rows 16 warp + (lane & 15), k-offset 8 (lane >> 4); B (W1 [k][n], transposed)
    // k-rows (lane & 15) of n-tile pair (lane >> 4)
    const uint32_t a_off = (uint32_t)((16 * warp + (lane & 15)) * WXLD + (lane >> 4) * 16);
    const uint32_t b_off = (uint32_t)(WXS_BYTES + (lane & 15) * WLD + (lane >> 4) * 16);
    int stage = 0;
    for (int s = 0; s < nsl; ++s) {
        cp_async_wait<WNST - 2>();
        __syncthreads();
        if (s + WNST - 1 < nsl) issue(stage == 0 ? WNST - 1 : stage - 1);
        cp_async_commit();
        const uint32_t st = sbase + (uint32_t)stage * WST_BYTES;
        const int kn = min(WKC, D - kcur) / 16;     // k-steps of this slice (D % 16 == 0)
        for (int kk = 0; kk < kn; ++kk) {
            uint32_t a[4], b[2][4];
            ldsm_x4(st + a_off + (uint32_t)(kk * 32), a);
            ldsm_x4_t(st + b_off + (uint32_t)(kk * 16 * WLD), b[0]);        // n-tiles 0, 1
            ldsm_x4_t(st + b_off + (uint32_t)(kk * 16 * WLD) + 32, b[1]);   // n-tiles 2, 3
#pragma unroll
            for (int n = 0; n < 4; ++n) mma16816(acc[n], a, b[n >> 1][(n & 1) * 2], b[n >> 1][(n & 1) * 2 + 1]);
        }
        kcur = kcur + WKC >= nsl * WKC ? 0 : kcur + WKC;
        stage = stage + 1 == WNST ? 0 : stage + 1;
    }
    cp_async_wait<0>();
    {   // SiLU of this warp's 16 x 32 product (rows 16 warp + g and + 8, columns 8 n + 2 t4 and + 1)
        const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = 16 * warp + g + (e >= 2 ? 8 : 0), c = 8 * n + 2 * t4 + (e & 1);
                const float z = acc[n][e];
                hs[r * HLD + c] = z / (1.0f + expf(-z));
            }
    }
    __syncthreads();
    if (tg >= ng) return;
    float w2[HID];
#pragma unroll
    for (int r = 0; r < HID / 2; ++r) {
        w2[2 * r] = __uint_as_float(w2p[r] << 16);
        w2[2 * r + 1] = __uint_as_float(w2p[r] & 0xffff0000u);
    }
    const int nrows = (int)(N - r0 < WGT ? N - r0 : WGT);
    for (int t = tg; t < nrows; t += ng) {
        const float4* hr = reinterpret_cast<const float4*>(hs + t * HLD);
        float a = 0.f;
#pragma unroll
        for (int r4 = 0; r4 < HID / 4; ++r4) {
            const float4 hv = hr[r4];
            a = fmaf(hv.x, w2[4 * r4], a);
            a = fmaf(hv.y, w2[4 * r4 + 1], a);
            a = fmaf(hv.z, w2[4 * r4 + 2], a);
            a = fmaf(hv.w, w2[4 * r4 + 3], a);
        }
        taps[(r0 + t) * HW4 + col] = a;
    }
}

}  // namespace kgen
}  // namespace jet
