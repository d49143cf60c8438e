// K2 (tensor-core form): chunked Gated DeltaNet prefill on tcgen05 / TMA.
//
// Gated delta rule (Jet-Nemotron paper, section 2.3) in chunked WY / UT form.
// Within a chunk of C = 64 tokens (r, i index tokens; s = state row = value
// channel; j = key feature):
//   G_r = sum_{t<=r} g_t,  gam_r = exp(G_r),  d_i = exp(G_{L-1} - G_i)
//   A_ri = b_r exp(G_r - G_i) k^_r.k^_i (i<r),  P_ri = exp(G_r - G_i) q^_r.k^_i (i<=r)
//   T = (I + A)^-1,  U = T diag(b) V,  W = T diag(b gam) K^
//   Wt = U - W S^T                                   (per-token residual values)
//   O  = diag(gam) Q^ S^T + P Wt
//   S <- gam_{L-1} S + Wt^T diag(d) K^
// Everything is arranged so the state row index is the MMA M dimension
// (M = 128 rows of S per CTA) and every product is one tcgen05 MMA family:
//   P1  [K;Q] K^T      -> TMEM XP (rows 0..63 = KK^T, 64..127 = QK^T)   M128 N64  K=dk
//   P2a V^T T1^T       -> TMEM X1 = U^T     (T1 = T diag(b))            M128 N64  K=64
//   P2b K^T T2^T       -> TMEM XW = W^T     (T2 = T diag(b gam/|k|))    M128 N64  K=64
//   P3  X1 -= S W^T    -> X1 = Wt^T                                     M128 N64  K=dk
//   P5a S Q^T          -> TMEM X2                                       M128 N64  K=dk
//   P4  S += (Wt^T diag(d/|k|)) K  (state accumulates in TMEM)          M128 Ndk  K=64
//   P5b Wt^T P^T       -> TMEM X3                                       M128 N64  K=64
//   o_r = gam_r / |q_r| X2[:, r] + X3[:, r]
// The L2 norms of q and k are folded into per-token scale factors, so the raw
// bf16 q / k / v tiles from TMA serve directly as MMA operands. The float32
// state lives in TMEM for the whole sequence; its bf16 copy is the A operand
// of P3 / P5a. The UT inverse (I + A)^-1 is computed in float32 on the CUDA
// cores by recursive doubling over 16 x 16 blocks. Decay factors are formed
// as exp(G_r - G_i) <= 1.
//
// One CTA = (sequence, head, 128 state rows); 128 threads; thread 0 issues
// TMA and MMA; the four warps read TMEM lanes 32w..32w+31 in the epilogues.
// The chunk's TMA tiles are double-buffered (chunk c+1 loads during chunk c).
// Every mbarrier wait is bounded; on expiry the CTA flags the device error
// word, drains what it issued (bounded), frees TMEM and returns.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "sm100.cuh"

namespace jet {
namespace pftc {

using namespace sm100;

constexpr int C = 64;
constexpr int ROWS = 128;
constexpr int THREADS = 128;
constexpr float EPS = 1e-6f;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t STAGE_BYTES = 49152;                 // KQ (2 x [K 8K | Q 8K]) + V (2 x 8K)
constexpr uint32_t OFF_KQ = 0, OFF_V = 32768;
constexpr uint32_t OFF_P = 2 * STAGE_BYTES;             // 8K  P [64 r][64 i] K-major
constexpr uint32_t OFF_T1 = OFF_P + 8192;               // 8K
constexpr uint32_t OFF_T2 = OFF_T1 + 8192;              // 8K
constexpr uint32_t OFF_WT = OFF_T2 + 8192;              // 16K W^T [128 features][64 tokens]
constexpr uint32_t OFF_AS = OFF_WT + 16384;             // 32K bf16 S, K-major, 2 x [128 x 64]
constexpr uint32_t OFF_AW = OFF_AS + 32768;             // 16K Wt^T
constexpr uint32_t OFF_AWD = OFF_AW + 16384;            // 16K Wt^T diag(d/|k|)
constexpr uint32_t OFF_AF = OFF_AS;                     // fp32 A [64][65] (aliases AS..AWD)
constexpr uint32_t OFF_TF = OFF_AS + 64 * 65 * 4;       // fp32 T [64][65]
constexpr uint32_t OFF_XB = OFF_TF + 64 * 65 * 4;       // fp32 block products (1024 floats)
constexpr uint32_t OFF_VEC = OFF_AWD + 16384;           // per-token vectors, 8 x 64 floats
constexpr uint32_t OFF_BAR = OFF_VEC + 2048;
constexpr uint32_t OFF_TSLOT = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = OFF_TSLOT + 64 + 1024;  // + alignment slack
static_assert(OFF_XB + 1024 * 4 <= OFF_VEC, "fp32 scratch overflows its alias region");

// TMEM columns
constexpr uint32_t TM_S = 0, TM_X1 = 128, TM_X2 = 192, TM_X3 = 256, TM_XP = 320, TM_XW = 384;
constexpr uint32_t TM_COLS = 512;

// per-token vectors of a chunk; G is kept in log2 units (G * log2 e) so that
// every decay factor is one exp2 of a difference
struct Vecs {
    float* G; float* gam; float* dcy; float* bet; float* ik; float* iq; float* graw;
};
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
// write 64 floats as one 128-byte SW128 row (8 chunks of 8 bf16)
__device__ __forceinline__ void st_row64(uint8_t* tile, int row, const float* v) {
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 u = make_uint4(pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]), pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                             pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]), pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
        *reinterpret_cast<uint4*>(tile + sw128_off(row, ch * 16)) = u;
    }
}
// sum of squares of one 64-wide SW128 row (bf16)
__device__ __forceinline__ float row_sumsq(const uint8_t* tile, int row, int nchunks) {
    float s = 0.f;
    for (int ch = 0; ch < nchunks; ++ch) {
        const uint4 u = *reinterpret_cast<const uint4*>(tile + sw128_off(row, ch * 16));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
            s += lo * lo + hi * hi;
        }
    }
    return s;
}

// T = (I + A)^-1 for strictly lower A [64][65] (fp32) by recursive doubling:
// invert the four 16 x 16 diagonal blocks by forward substitution (one thread
// per column, the column held in registers), then merge pairs with
//   [[T11, 0], [X, T22]],  X = -T22 A21 T11
// at 16 -> 32 and 32 -> 64. Every loop has a constant trip count and several
// independent accumulators, so the shared-memory loads pipeline. Xs holds
// 1024 floats of scratch.
__device__ __forceinline__ void invert_unit_lower(const float* A, float* T, float* Xs, int tid) {
    if (tid < 64) {
        const int c = tid, j = c >> 4, cl = c & 15;
        const float* Ab = A + (j * 16) * 65 + j * 16;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float x = (r == cl) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) x -= Ab[r * 65 + i] * t[i];
            t[r] = x;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T[(j * 16 + r) * 65 + c] = t[r];
    } else {
        // zero the strictly upper off-diagonal blocks: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
        for (int e = tid - 64; e < 6 * 256; e += 64) {
            const int blk = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            T[(bi * 16 + rr) * 65 + bj * 16 + cc] = 0.f;
        }
    }
    __syncthreads();
    // 16 -> 32: pairs (b1, b0) = (1, 0) and (3, 2); thread: column c, rows rg*4 .. rg*4+3
    const int pr = tid >> 6, c16 = tid & 15, rg = (tid >> 4) & 3;
    const int b0 = pr * 2, b1 = b0 + 1;
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float tv = T[(b0 * 16 + k) * 65 + b0 * 16 + c16];
#pragma unroll
            for (int m = 0; m < 4; ++m) acc[m] += A[(b1 * 16 + rg * 4 + m) * 65 + b0 * 16 + k] * tv;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) Xs[pr * 256 + (rg * 4 + m) * 16 + c16] = acc[m];
    }
    __syncthreads();
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float xv = Xs[pr * 256 + k * 16 + c16];
#pragma unroll
            for (int m = 0; m < 4; ++m) acc[m] += T[(b1 * 16 + rg * 4 + m) * 65 + b1 * 16 + k] * xv;
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) T[(b1 * 16 + rg * 4 + m) * 65 + b0 * 16 + c16] = -acc[m];
    }
    __syncthreads();
    // 32 -> 64: thread: column c, rows rb .. rb+7 of the lower-left 32 x 32 block
    const int c32 = tid & 31, rb = (tid >> 5) * 8;
    {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float tv = T[k * 65 + c32];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] += A[(32 + rb + m) * 65 + k] * tv;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) Xs[(rb + m) * 32 + c32] = acc[m];
    }
    __syncthreads();
    {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float xv = Xs[k * 32 + c32];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] += T[(32 + rb + m) * 65 + 32 + k] * xv;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) T[(32 + rb + m) * 65 + c32] = -acc[m];
    }
    __syncthreads();
}

template <int DK>
__global__ void __launch_bounds__(THREADS, 1)
gdn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
                      const float* __restrict__ beta, const float* S0, __nv_bfloat16* __restrict__ o,
                      float* S_out, int Tn, int H, int dv) {
    static_assert(DK % 32 == 0 && DK >= 64 && DK <= 128, "DK in {64, 96, 128}");
    constexpr int NKB = (DK + 63) / 64;                  // 64-wide column blocks of q / k
    constexpr int KSTEPS = DK / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BAR);       // [2]
    uint64_t* mbar = full + 2;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + OFF_TSLOT);
    float* vec = reinterpret_cast<float*>(sm + OFF_VEC);
    Vecs V{vec, vec + 64, vec + 128, vec + 192, vec + 256, vec + 320, vec + 384};
    float* AF = reinterpret_cast<float*>(sm + OFF_AF);
    float* TF = reinterpret_cast<float*>(sm + OFF_TF);
    float* XB = reinterpret_cast<float*>(sm + OFF_XB);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int c0 = blockIdx.x * ROWS, h = blockIdx.y, b = blockIdx.z;
    const long long bh = (long long)b * H + h;
    const int nch = (Tn + C - 1) / C;
    const uint32_t tx_bytes = (uint32_t)(NKB * 2 * 8192 + 2 * 8192);

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(mbar, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) tmem_alloc(tslot, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tslot;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    // ---- initial state into TMEM (row tid of the slice)
    {
        const float* src = S0 ? S0 + (bh * dv + c0 + tid) * DK : nullptr;
#pragma unroll
        for (int cb = 0; cb < DK / 32; ++cb) {
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = src ? __float_as_uint(src[cb * 32 + j]) : 0u;
            tmem_st32(tb + lane_base + TM_S + cb * 32, r);
        }
        tmem_st_wait();
    }

    auto issue_loads = [&](int c, int s) {
        uint8_t* st = sm + s * STAGE_BYTES;
        const int z = (int)((long long)b * Tn + (long long)c * C);
        mbar_expect_tx(&full[s], tx_bytes);
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
            tma_load_3d(st + OFF_KQ + kb * 16384, &tm_k, &full[s], kb * 64, h, z);
            tma_load_3d(st + OFF_KQ + kb * 16384 + 8192, &tm_q, &full[s], kb * 64, h, z);
        }
        tma_load_3d(st + OFF_V, &tm_v, &full[s], c0, h, z);
        tma_load_3d(st + OFF_V + 8192, &tm_v, &full[s], c0 + 64, h, z);
    };
    if (tid == 0) issue_loads(0, 0);

    uint32_t full_par[2] = {0u, 0u};
    uint32_t mma_par = 0u;
    bool ok = true;
    int issued_next = 0;        // thread 0: a load for chunk c+1 is in flight

    for (int c = 0; c < nch && ok; ++c) {
        const int s = c & 1;
        uint8_t* st = sm + s * STAGE_BYTES;
        uint8_t* KQ = st + OFF_KQ;
        const int t0 = c * C;
        const int L = min(C, Tn - t0);
        issued_next = 0;
        if (tid == 0 && c + 1 < nch) { issue_loads(c + 1, s ^ 1); issued_next = 1; }

        if (tid < C) {
            const long long off = ((long long)b * Tn + t0 + tid) * H + h;
            V.graw[tid] = tid < L ? g[off] : 0.f;
            V.bet[tid] = tid < L ? beta[off] : 0.f;
        }
        ok = mbar_wait(&full[s], full_par[s]);
        full_par[s] ^= 1u;
        // L2 norms of the k rows (threads 0..63) and q rows (64..127)
        {
            const int r = tid & 63;
            const uint32_t qoff = tid < 64 ? 0u : 8192u;
            float ss = 0.f;
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                const int nck = (DK - kb * 64) >= 64 ? 8 : (DK - kb * 64) / 8;
                ss += row_sumsq(KQ + kb * 16384 + qoff, r, nck);
            }
            const float inv = 1.0f / sqrtf(ss + EPS);
            if (tid < 64) V.ik[r] = inv; else V.iq[r] = inv;
        }
        __syncthreads();
        if (warp == 0) {        // inclusive scan of the 64 gates, two per lane
            const int l = tid;
            float a0 = V.graw[2 * l], a1 = a0 + V.graw[2 * l + 1];
            float run = a1;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, run, o2);
                if (l >= o2) run += y;
            }
            const float excl = run - a1;
            V.G[2 * l] = (excl + a0) * LOG2E;
            V.G[2 * l + 1] = run * LOG2E;
        }
        __syncthreads();
        if (tid < C) {
            V.gam[tid] = exp2f(V.G[tid]);
            V.dcy[tid] = tid < L ? exp2f(V.G[L - 1] - V.G[tid]) : 0.f;
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;

        // ---- P1: [K;Q] K^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t kq = smem_u32(KQ);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16_ss(tb + TM_XP, sw128_desc(kq + off, 16, 1024), sw128_desc(kq + off, 16, 1024),
                            idesc_bf16(128, 64, false, false), kk > 0);
            }
            mma_commit(mbar);
        }
        ok = mbar_wait(mbar, mma_par);
        mma_par ^= 1u;
        tc_fence_after();
        // ---- E1: A (fp32) from KK^T rows, P (bf16 tile) from QK^T rows
        {
            uint32_t x[64];
            tmem_ld32(tb + lane_base + TM_XP, x);
            tmem_ld32(tb + lane_base + TM_XP + 32, x + 32);
            tmem_ld_wait();
            const int r = tid & 63;
            const float Gr = V.G[r];
            if (tid < 64) {
                const float sc = V.bet[r] * V.ik[r];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    AF[r * 65 + i] = i < r ? sc * exp2f(Gr - V.G[i]) * __uint_as_float(x[i]) * V.ik[i] : 0.f;
            } else {
                const float sc = V.iq[r];
                float p[64];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    p[i] = i <= r ? sc * exp2f(Gr - V.G[i]) * __uint_as_float(x[i]) * V.ik[i] : 0.f;
                st_row64(sm + OFF_P, r, p);
            }
        }
        __syncthreads();
        // ---- E2: T = (I + A)^-1, then T1 = T diag(b), T2 = T diag(b gam / |k|)
        invert_unit_lower(AF, TF, XB, tid);
        {
            const int r = tid >> 1, half = tid & 1;
            float t1[32], t2[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = half * 32 + e;
                const float tv = i <= r ? TF[r * 65 + i] : 0.f;
                t1[e] = tv * V.bet[i];
                t2[e] = tv * V.bet[i] * V.gam[i] * V.ik[i];
            }
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int cb = half * 64 + ch * 16;          // byte column within the 128-byte row
                uint4 u1 = make_uint4(pack_bf16x2(t1[8 * ch], t1[8 * ch + 1]), pack_bf16x2(t1[8 * ch + 2], t1[8 * ch + 3]),
                                      pack_bf16x2(t1[8 * ch + 4], t1[8 * ch + 5]), pack_bf16x2(t1[8 * ch + 6], t1[8 * ch + 7]));
                uint4 u2 = make_uint4(pack_bf16x2(t2[8 * ch], t2[8 * ch + 1]), pack_bf16x2(t2[8 * ch + 2], t2[8 * ch + 3]),
                                      pack_bf16x2(t2[8 * ch + 4], t2[8 * ch + 5]), pack_bf16x2(t2[8 * ch + 6], t2[8 * ch + 7]));
                *reinterpret_cast<uint4*>(sm + OFF_T1 + sw128_off(r, cb)) = u1;
                *reinterpret_cast<uint4*>(sm + OFF_T2 + sw128_off(r, cb)) = u2;
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- P2a: U^T = V^T T1^T ;  P2b: W^T = K^T T2^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t v = smem_u32(st + OFF_V), kq = smem_u32(KQ);
            const uint32_t t1 = smem_u32(sm + OFF_T1), t2 = smem_u32(sm + OFF_T2);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tb + TM_X1, sw128_desc(v + kk * 2048, 8192, 1024), sw128_desc(t1 + kk * 32, 16, 1024),
                            idesc_bf16(128, 64, true, false), kk > 0);
                mma_bf16_ss(tb + TM_XW, sw128_desc(kq + kk * 2048, 16384, 1024), sw128_desc(t2 + kk * 32, 16, 1024),
                            idesc_bf16(128, 64, true, false), kk > 0);
            }
            mma_commit(mbar);
        }
        ok = mbar_wait(mbar, mma_par);
        mma_par ^= 1u;
        tc_fence_after();
        // ---- E3: W^T rows (feature j = tid) -> bf16 MN-major tile; E4: S -> bf16 A operand, S <- gam_L S
        {
            uint32_t x[64];
            tmem_ld32(tb + lane_base + TM_XW, x);
            tmem_ld32(tb + lane_base + TM_XW + 32, x + 32);
            tmem_ld_wait();
            if (tid < DK) {
                float w[64];
#pragma unroll
                for (int i = 0; i < 64; ++i) w[i] = __uint_as_float(x[i]);
                st_row64(sm + OFF_WT, tid, w);
            }
        }
        {
            const float gL = V.gam[L - 1];
#pragma unroll
            for (int cb = 0; cb < DK / 32; ++cb) {
                uint32_t x[32];
                tmem_ld32(tb + lane_base + TM_S + cb * 32, x);
                tmem_ld_wait();
                // 32 columns = half of a 64-wide block: 4 chunks of 8
                uint8_t* tile = sm + OFF_AS + (cb >> 1) * 16384;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int colb = ((cb & 1) * 32 + ch * 8) * 2;
                    uint4 u = make_uint4(pack_bf16x2(__uint_as_float(x[8 * ch]), __uint_as_float(x[8 * ch + 1])),
                                         pack_bf16x2(__uint_as_float(x[8 * ch + 2]), __uint_as_float(x[8 * ch + 3])),
                                         pack_bf16x2(__uint_as_float(x[8 * ch + 4]), __uint_as_float(x[8 * ch + 5])),
                                         pack_bf16x2(__uint_as_float(x[8 * ch + 6]), __uint_as_float(x[8 * ch + 7])));
                    *reinterpret_cast<uint4*>(tile + sw128_off(tid, colb)) = u;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = __float_as_uint(gL * __uint_as_float(x[j]));
                tmem_st32(tb + lane_base + TM_S + cb * 32, x);
            }
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- P3: X1 -= S W^T (-> Wt^T) ; P5a: X2 = S Q^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t as = smem_u32(sm + OFF_AS), wt = smem_u32(sm + OFF_WT), kq = smem_u32(KQ);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint64_t a = sw128_desc(as + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                mma_bf16_ss(tb + TM_X1, a, sw128_desc(wt + kk * 2048, 8192, 1024),
                            idesc_bf16(128, 64, false, true, true), 1);
                mma_bf16_ss(tb + TM_X2, a, sw128_desc(kq + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                            idesc_bf16(128, 64, false, false), kk > 0);
            }
            mma_commit(mbar);
        }
        ok = mbar_wait(mbar, mma_par);
        mma_par ^= 1u;
        tc_fence_after();
        // ---- E5: Wt^T -> bf16 (as is, and scaled by d/|k| per token)
        {
            uint32_t x[64];
            tmem_ld32(tb + lane_base + TM_X1, x);
            tmem_ld32(tb + lane_base + TM_X1 + 32, x + 32);
            tmem_ld_wait();
            float w[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) w[i] = __uint_as_float(x[i]);
            st_row64(sm + OFF_AW, tid, w);
#pragma unroll
            for (int i = 0; i < 64; ++i) w[i] *= V.dcy[i] * V.ik[i];
            st_row64(sm + OFF_AWD, tid, w);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- P4: S += (Wt^T diag(d/|k|)) K ;  P5b: X3 = Wt^T P^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t awd = smem_u32(sm + OFF_AWD), aw = smem_u32(sm + OFF_AW);
            const uint32_t kq = smem_u32(KQ), p = smem_u32(sm + OFF_P);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16_ss(tb + TM_S, sw128_desc(awd + kk * 32, 16, 1024), sw128_desc(kq + kk * 2048, 16384, 1024),
                            idesc_bf16(128, DK, false, true), 1);
                mma_bf16_ss(tb + TM_X3, sw128_desc(aw + kk * 32, 16, 1024), sw128_desc(p + kk * 32, 16, 1024),
                            idesc_bf16(128, 64, false, false), kk > 0);
            }
            mma_commit(mbar);
        }
        ok = mbar_wait(mbar, mma_par);
        mma_par ^= 1u;
        tc_fence_after();
        // ---- E6: o_r = gam_r/|q_r| X2[:, r] + X3[:, r], staged as a [64 token][128 channel]
        // bf16 tile, then written with 16-byte coalesced stores
        {
            __nv_bfloat16* ot = reinterpret_cast<__nv_bfloat16*>(sm + OFF_AW);
            uint32_t x2[32], x3[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tb + lane_base + TM_X2 + half * 32, x2);
                tmem_ld32(tb + lane_base + TM_X3 + half * 32, x3);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int r = half * 32 + j;
                    ot[r * ROWS + tid] = __float2bfloat16_rn(V.gam[r] * V.iq[r] * __uint_as_float(x2[j]) +
                                                             __uint_as_float(x3[j]));
                }
            }
            __syncthreads();
            const long long tstride = (long long)H * dv;
            __nv_bfloat16* obase = o + ((long long)b * Tn + t0) * tstride + (long long)h * dv + c0;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int q = tid + m * THREADS, r = q >> 4, ch = q & 15;
                if (r < L)
                    *reinterpret_cast<uint4*>(obase + r * tstride + ch * 8) =
                        *reinterpret_cast<const uint4*>(ot + r * ROWS + ch * 8);
            }
        }
        tc_fence_before();
        ok = __syncthreads_and(ok);
    }

    if (ok) {
        // ---- final state out
        float* dst = S_out + (bh * dv + c0 + tid) * DK;
#pragma unroll
        for (int cb = 0; cb < DK / 32; ++cb) {
            uint32_t x[32];
            tmem_ld32(tb + lane_base + TM_S + cb * 32, x);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(dst + cb * 32 + j) =
                    make_float4(__uint_as_float(x[j]), __uint_as_float(x[j + 1]), __uint_as_float(x[j + 2]),
                                __uint_as_float(x[j + 3]));
        }
    } else if (tid == 0) {
        // a wait ran out: drain what this CTA issued (bounded) before freeing TMEM
        mbar_wait(mbar, mma_par);
        if (issued_next) mbar_wait(&full[0], full_par[0]), mbar_wait(&full[1], full_par[1]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tb, TM_COLS);
}

}  // namespace pftc
}  // namespace jet
