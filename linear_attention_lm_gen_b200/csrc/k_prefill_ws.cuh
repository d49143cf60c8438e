// K2 (tensor-core, warp-specialised): chunked Gated DeltaNet prefill.
//
// Gated delta rule (Jet-Nemotron paper, section 2.3) in chunked WY / UT form.
// Within a chunk of C = 64 tokens (r, i index tokens; the state row index is
// the value channel; j = key feature):
//   G_r = sum_{t<=r} g_t,  gam_r = exp(G_r),  d_i = exp(G_{L-1} - G_i)
//   A_ri = b_r exp(G_r - G_i) k^_r.k^_i (i<r),  P_ri = exp(G_r - G_i) q^_r.k^_i (i<=r)
//   T = (I + A)^-1,  U = T diag(b) V,  W = T diag(b gam) K^
//   Wt = U - W S^T                                   (per-token residual values)
//   O  = diag(gam) Q^ S^T + P Wt
//   S <- gam_{L-1} S + Wt^T diag(d) K^
// The L2 norms of q and k are folded into per-token scales, so the raw bf16
// q / k / v tiles from TMA serve directly as MMA operands; the float32 state
// lives in TMEM for the whole sequence (its bf16 copy is the A operand of the
// state products). Decay factors are formed as exp(G_r - G_i) <= 1 (the lower
// left 32 x 32 block as a product of two factors that are each <= 1), never
// as a ratio of exponentials. The UT inverse runs in float32 on the CUDA
// cores (16 x 16 diagonal blocks) and tf32 warp MMAs (the 16->32->64 merges).
// One CTA = (sequence, head, 128 state rows); the state-independent work of
// chunk c+1 overlaps the state chain of chunk c:
//
//   warps 0-3   CHAIN  E4: S (TMEM) -> bf16 copy + S <- gam_L S;  E5: Wt^T ->
//                      bf16 (plain and scaled by d/|k|);  E6: O -> global
//   warps 4-11  PREP   norms, cumulative gates, A and P from P1, the UT
//                      inverse, T1 / T2, Q~ = diag(gam/|q|) Q in place, W^T
//   warp  12    CTRL   one thread: every TMA load and tcgen05 MMA, in a fixed
//                      dependency-ordered schedule
//
// MMA families per chunk (M = 128 state rows, TMEM accumulators):
//   P1  [K;Q] K^T          -> XP      (prep)
//   P2a V^T T1^T           -> X1[c&1] (U^T)      P2b K^T T2^T -> XW (W^T)
//   P3  X1 -= S W^T        -> Wt^T    (chain)    P5a S Q~^T   -> X2[c&1]
//   P4  S += (Wt^T diag(d/|k|)) K                P5b X2 += Wt^T P^T
// With Q~ pre-scaled, X2 holds O^T directly.
//
// Buffers: K/Q tiles double-buffered (Q is overwritten in place by Q~ once
// P1 has read it), V single, P double, T1/T2/W^T single, bf16 S copy and Wt^T
// copies owned by the chain; TMEM: S, X1[2], X2[2], XP, XW = 512 columns.
// Every wait is bounded; a timed-out thread raises a CTA-wide abort flag so
// the others stop waiting, then the control thread drains its commits and
// TMEM is freed.
#pragma once
#include "k_prefill_common.cuh"

namespace jet {
namespace pfws {

constexpr int NCHAIN = 128;
constexpr int THREADS = NCHAIN + NPREP + 32;          // 416
constexpr int PREP0 = NCHAIN, CTRL0 = NCHAIN + NPREP;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;                         // [2] x 32K: per 64-col block [K 8K | Q 8K]
constexpr uint32_t OFF_V = 65536;                      // 16K: 2 x [64 tok x 64 ch]
constexpr uint32_t OFF_P = 81920;                      // [2] x 8K
constexpr uint32_t OFF_T1 = 98304, OFF_T2 = 106496;    // 8K each
constexpr uint32_t OFF_WT = 114688;                    // 16K  W^T [128 features][64 tokens]
constexpr uint32_t OFF_AS = 131072;                    // 32K  bf16 S [128][dk]
constexpr uint32_t OFF_AW = 163840;                    // 16K  Wt^T
constexpr uint32_t OFF_AWD = 180224;                   // 16K  Wt^T diag(d/|k|); output staging alias
constexpr uint32_t OFF_AF = 196608;                    // 64 x 68 fp32, A then T in place
constexpr uint32_t OFF_XS = OFF_AF + 64 * LDA * 4;     // 32 x 40 fp32 block products
constexpr uint32_t OFF_VEC = OFF_XS + 32 * LDX * 4;    // [2] x 8 x 64 fp32
constexpr uint32_t OFF_PN = OFF_VEC + 4096;            // 2 x 128 fp32 partial norms
constexpr uint32_t OFF_BAR = OFF_PN + 1024;            // mbarriers
constexpr uint32_t OFF_TSLOT = OFF_BAR + 256;
constexpr uint32_t OFF_ABORT = OFF_TSLOT + 16;
constexpr uint32_t SMEM_BYTES = OFF_ABORT + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t TM_S = 0, TM_X1 = 128, TM_X2 = 256, TM_XP = 384, TM_XW = 448, TM_COLS = 512;

// mbarrier indices
enum {
    B_KFULL = 0,      // [2] TMA K/Q tiles landed
    B_VFULL = 2,      // TMA V tile landed
    B_P1 = 3,         // P1 complete
    B_P2 = 4,         // P2a/P2b complete
    B_P3 = 5,         // P3/P5a complete
    B_SDONE = 6,      // [2] P4/P5b complete
    B_VEC = 8,        // [2] per-token vectors written (prep)
    B_TREADY = 10,    // T1/T2 written (prep)
    B_WQ = 11,        // W^T and Q~ written (prep)
    B_AS = 12,        // bf16 S written, S scaled (chain)
    B_AW = 13,        // Wt^T copies written (chain)
    B_X1FREE = 14,    // [2] X1 read by E5 (chain)
    B_X2FREE = 16,    // [2] X2 read by E6 (chain)
    NBARS = 18
};

__device__ __forceinline__ Vec vec_at(uint8_t* sm, int p) {
    return vec_from(reinterpret_cast<float*>(sm + OFF_VEC) + p * 512);
}

template <int DK>
__global__ void __launch_bounds__(THREADS, 1)
gdn_prefill_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ g,
                      const float* __restrict__ beta, const float* S0, __nv_bfloat16* __restrict__ o,
                      float* S_out, int Tn, int H, int dv, const Seg seg) {
    static_assert(DK % 32 == 0 && DK >= 64 && DK <= 128, "DK in {64, 96, 128}");
    constexpr int NKB = (DK + 63) / 64;
    constexpr int KSTEPS = DK / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + OFF_TSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_ABORT);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int ns = dv / ROWS;
    const int h = blockIdx.y, b = blockIdx.z / seg.zseg, p_seg = blockIdx.z % seg.zseg;
    const bool trans = blockIdx.x == ns;                  // transition slice (phase A, p >= 1)
    if (trans && (!seg.phaseA || p_seg == 0)) return;     // whole CTA, before any barrier
    const int c0 = blockIdx.x * ROWS;                     // transition slice: past dv, V reads as zero
    const long long bh = (long long)b * H + h;
    const int tbeg = p_seg * seg.seg_chunks * C;
    const int tend = min(Tn, tbeg + seg.seg_chunks * C);
    const int nch = (tend - tbeg + C - 1) / C;
    const bool write_o = !seg.phaseA;

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (tid == CTRL0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) tmem_alloc(tslot, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tslot;
    pdl_wait();                                           // inputs are read from here on
    pdl_trigger();

    if (warp < 4) {
        // =============================================================== CHAIN
        const int ct = tid;
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        {   // initial state (row ct of the slice)
            const float* src = nullptr;
            if (!seg.phaseA && seg.nseg > 1) {
                src = seg.Sst + ((((long long)b * seg.nseg + p_seg) * H + h) * dv + c0 + ct) * DK;
            } else if (p_seg == 0 && !trans && S0) {
                src = S0 + (bh * dv + c0 + ct) * DK;
            }
#pragma unroll
            for (int cb = 0; cb < DK / 32; ++cb) {
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    r[j] = trans ? (cb * 32 + j == ct ? 0x3f800000u : 0u) : (src ? __float_as_uint(src[cb * 32 + j]) : 0u);
                tmem_st32(tb + lb + TM_S + cb * 32, r);
            }
            tmem_st_wait();
        }
        auto emit_output = [&](int cc) {   // E6 for chunk cc: X2 -> staging -> global
            if (!write_o) {
                named_sync(2, NCHAIN);
                if (ct == 0) arrive(&bars[B_X2FREE + (cc & 1)]);
                return;
            }
            __nv_bfloat16* ot = reinterpret_cast<__nv_bfloat16*>(sm + OFF_AWD);
            const uint32_t x2 = TM_X2 + (uint32_t)(cc & 1) * 64;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t x[32];
                tmem_ld32(tb + lb + x2 + half * 32, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) ot[(half * 32 + j) * ROWS + ct] = __float2bfloat16_rn(__uint_as_float(x[j]));
            }
            tc_fence_before();
            named_sync(2, NCHAIN);
            if (ct == 0) arrive(&bars[B_X2FREE + (cc & 1)]);
            const int t0 = tbeg + cc * C, L = min(C, tend - t0);
            const long long tstride = (long long)H * dv;
            __nv_bfloat16* obase = o + ((long long)b * Tn + t0) * tstride + (long long)h * dv + c0;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int qd = ct + m * NCHAIN, r = qd >> 4, ch = qd & 15;
                if (r < L)
                    *reinterpret_cast<uint4*>(obase + r * tstride + ch * 8) =
                        *reinterpret_cast<const uint4*>(ot + r * ROWS + ch * 8);
            }
            named_sync(2, NCHAIN);
        };
        for (int c = 0; c < nch; ++c) {
            const int p = c & 1;
            Vec V = vec_at(sm, p);
            bool okw = c < 1 || wait_bar(&bars[B_SDONE + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag);
            okw = okw && wait_bar(&bars[B_VEC + p], (c >> 1) & 1, abort_flag);
            if (!group_all(2, NCHAIN, okw)) break;
            tc_fence_after();
            // ---- E4: S -> bf16 copy, S <- gam_L S
            {
                const int L = min(C, tend - (tbeg + c * C));
                const float gL = V.gam[L - 1];
#pragma unroll
                for (int cb = 0; cb < DK / 32; ++cb) {
                    uint32_t x[32];
                    tmem_ld32(tb + lb + TM_S + cb * 32, x);
                    tmem_ld_wait();
                    uint8_t* tile = sm + OFF_AS + (cb >> 1) * 16384;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(x[8 * ch + e]);
                        *reinterpret_cast<uint4*>(tile + sw128_off(ct, ((cb & 1) * 32 + ch * 8) * 2)) = pack8(f);
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = __float_as_uint(gL * __uint_as_float(x[j]));
                    tmem_st32(tb + lb + TM_S + cb * 32, x);
                }
                tmem_st_wait();
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NCHAIN);
            if (ct == 0) arrive(&bars[B_AS]);
            // ---- E6 of the previous chunk while P3 / P5a run
            if (c >= 1) emit_output(c - 1);
            // ---- E5: Wt^T -> bf16 (plain and scaled by d/|k|)
            if (!group_all(2, NCHAIN, wait_bar(&bars[B_P3], c & 1, abort_flag))) break;
            tc_fence_after();
            {
                const uint32_t x1 = TM_X1 + (uint32_t)p * 64;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t x[32];
                    tmem_ld32(tb + lb + x1 + half * 32, x);
                    tmem_ld_wait();
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float f[8], fd[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int i = half * 32 + ch * 8 + e;
                            f[e] = __uint_as_float(x[ch * 8 + e]);
                            fd[e] = f[e] * V.dcy[i] * V.ik[i];
                        }
                        const uint32_t off = sw128_off(ct, (half * 32 + ch * 8) * 2);
                        *reinterpret_cast<uint4*>(sm + OFF_AW + off) = pack8(f);
                        *reinterpret_cast<uint4*>(sm + OFF_AWD + off) = pack8(fd);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NCHAIN);
            if (ct == 0) {
                arrive(&bars[B_AW]);
                arrive(&bars[B_X1FREE + p]);
            }
        }
        // last chunk: output and final state
        const bool fin = !*abort_flag && nch > 0 &&
                         wait_bar(&bars[B_SDONE + ((nch - 1) & 1)], ((nch - 1) >> 1) & 1, abort_flag);
        if (group_all(2, NCHAIN, fin)) {
            tc_fence_after();
            emit_output(nch - 1);
            float* dst = nullptr;
            if (seg.phaseA) {
                const long long bp = (long long)b * (seg.nseg - 1) + p_seg;
                if (trans) { if (ct < DK) dst = seg.Ao + ((bp * H + h) * DK + ct) * trans_ld(DK); }
                else dst = seg.Eo + ((bp * H + h) * dv + c0 + ct) * DK;
            } else if (p_seg == seg.nseg - 1) {
                dst = S_out + (bh * dv + c0 + ct) * DK;
            }
#pragma unroll
            for (int cb = 0; cb < DK / 32; ++cb) {
                if (!dst) break;
                uint32_t x[32];
                tmem_ld32(tb + lb + TM_S + cb * 32, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4*>(dst + cb * 32 + j) =
                        make_float4(__uint_as_float(x[j]), __uint_as_float(x[j + 1]), __uint_as_float(x[j + 2]),
                                    __uint_as_float(x[j + 3]));
            }
        }
    } else if (warp < 12) {
        // =============================================================== PREP
        const int pt = tid - PREP0;                 // 0..255 (warps 4-11: lane quarter = warp & 3)
        float* AF = reinterpret_cast<float*>(sm + OFF_AF);
        float* XS = reinterpret_cast<float*>(sm + OFF_XS);
        float* PN = reinterpret_cast<float*>(sm + OFF_PN);
        // per-token vectors of chunk cv into vec[cv & 1]; gb holds its g (pt < 64)
        // or beta (64 <= pt < 128), loaded one chunk ahead
        auto vec_phase = [&](int cv, float gb) -> bool {
            const int pv = cv & 1;
            const int t0 = tbeg + cv * C, L = min(C, tend - t0);
            uint8_t* KQ = sm + OFF_KQ + pv * 32768;
            Vec V = vec_at(sm, pv);
            // vec[pv] is free once E5 of chunk cv-2 has read it
            bool okw = cv < 2 || wait_bar(&bars[B_X1FREE + pv], ((cv - 2) >> 1) & 1, abort_flag);
            okw = okw && wait_bar(&bars[B_KFULL + pv], (cv >> 1) & 1, abort_flag);
            if (!group_all(1, NPREP, okw)) return false;
            prep_vectors<DK>(KQ, V, PN, gb, L, pt, 1);
            if (pt == 0) arrive(&bars[B_VEC + pv]);
            return true;
        };
        auto load_gb = [&](int cv) -> float {
            float v = 0.f;
            if (cv < nch && pt < 128) {
                const int r = pt & 63;
                if (r < min(C, tend - (tbeg + cv * C))) {
                    const long long off = ((long long)b * Tn + tbeg + cv * C + r) * H + h;
                    v = pt < 64 ? g[off] : beta[off];
                }
            }
            return v;
        };
        bool alive = vec_phase(0, load_gb(0));
        float gb_next = load_gb(1);
        for (int c = 0; c < nch && alive; ++c) {
            const int p = c & 1;
            uint8_t* KQ = sm + OFF_KQ + p * 32768;
            Vec V = vec_at(sm, p);
            // ---- E1: A (fp32, rows 0..63 of XP) and P (bf16 tile, rows 64..127)
            bool okw = c < 2 || wait_bar(&bars[B_SDONE + p], ((c - 2) >> 1) & 1, abort_flag);   // P[p] free
            okw = okw && wait_bar(&bars[B_P1], c & 1, abort_flag);
            if (!group_all(1, NPREP, okw)) break;
            tc_fence_after();
            prep_e1(tb + TM_XP, V, AF, sm + OFF_P + p * 8192, pt);
            named_sync(1, NPREP);
            // ---- UT inverse in place: 16x16 diagonal blocks, then 16 -> 32 -> 64 doubling
            ut_inverse(AF, XS, pt, 1);
            // ---- T1 = T diag(b), T2 = T diag(b gam / |k|): row r = pt >> 2, 16 columns
            prep_t1t2(AF, V, sm + OFF_T1, sm + OFF_T2, pt);
            fence_async_smem();
            tc_fence_before();
            named_sync(1, NPREP);
            if (pt == 0) arrive(&bars[B_TREADY]);
            // ---- Q~ = diag(gam / |q|) Q, in place (P1 has consumed Q)
            prep_qtilde<DK>(KQ, V, pt);
            // ---- next chunk's per-token vectors while P2 runs
            if (c + 1 < nch) {
                const float gbn = gb_next;
                gb_next = load_gb(c + 2);
                if (!vec_phase(c + 1, gbn)) break;
            }
            // ---- W^T (rows = features) once P3 of the previous chunk has read the old one
            okw = c < 1 || wait_bar(&bars[B_P3], (c - 1) & 1, abort_flag);
            okw = okw && wait_bar(&bars[B_P2], c & 1, abort_flag);
            if (!group_all(1, NPREP, okw)) break;
            tc_fence_after();
            prep_wt<DK>(tb + TM_XW, sm + OFF_WT, pt);
            fence_async_smem();
            tc_fence_before();
            named_sync(1, NPREP);
            if (pt == 0) arrive(&bars[B_WQ]);
        }
    } else if (tid == CTRL0) {
        // =============================================================== CTRL
        // One thread issues every TMA load and MMA in a fixed order that
        // follows the dependency graph of the two pipelines, blocking on the
        // one mbarrier each step needs (no cycle: every awaited event depends
        // only on actions issued earlier in this order):
        //   prologue: KQ(0) KQ(1) V(0) P1(0) P2(0) P1(1)
        //   chunk c:  P3(c) P4(c) KQ(c+2) V(c+1) P2(c+1) P1(c+2)
        // (P1(c+2) may start as soon as the prep group has read the P1(c+1)
        // result, i.e. once T1/T2 of c+1 exist, which P2(c+1) waited for)
        const uint32_t tx_kq = (uint32_t)(NKB * 2 * 8192);
        bool ok = true;
        // wait for `phase` (0-based) of mbarrier `bar`: non-blocking test with a
        // short sleep between polls (a woken try_wait costs ~300 cycles here)
        auto W = [&](int bar, int phase) {
            if (!ok) return false;
            const uint64_t t0 = global_ns();
            for (uint32_t i = 0;; ++i) {
                if (mbar_test_wait(&bars[bar], (uint32_t)phase & 1u)) return true;
                if ((i & 1023u) == 1023u) {
                    if (*abort_flag) { ok = false; return false; }
                    if (global_ns() - t0 > kWaitLimitNs) break;
                }
                __nanosleep(32);
            }
            *abort_flag = 1;
            flag_error(DEVERR_TIMEOUT);
            ok = false;
            return false;
        };
        auto load_kq = [&](int c) {
            const int sb = c & 1;
            uint8_t* dst = sm + OFF_KQ + sb * 32768;
            const int z = (int)((long long)b * Tn + tbeg + (long long)c * C);
            mbar_expect_tx(&bars[B_KFULL + sb], tx_kq);
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) {
                tma_load_3d(dst + kb * 16384, &tm_k, &bars[B_KFULL + sb], kb * 64, h, z);
                tma_load_3d(dst + kb * 16384 + 8192, &tm_q, &bars[B_KFULL + sb], kb * 64, h, z);
            }
        };
        auto load_v = [&](int c) {
            const int z = (int)((long long)b * Tn + tbeg + (long long)c * C);
            mbar_expect_tx(&bars[B_VFULL], 16384);
            tma_load_3d(sm + OFF_V, &tm_v, &bars[B_VFULL], c0, h, z);
            tma_load_3d(sm + OFF_V + 8192, &tm_v, &bars[B_VFULL], c0 + 64, h, z);
        };
        // descriptor bases: the start-address field is the low 14 bits of
        // (address >> 4), so an operand offset is added to the 64-bit value
        const uint64_t dK16 = sw128_desc(smem_u32(sm + OFF_KQ), 16, 1024);        // K-major, 1024 SBO
        const uint64_t dKmn = sw128_desc(smem_u32(sm + OFF_KQ), 16384, 1024);     // K tile as MN-major
        const uint64_t dV = sw128_desc(smem_u32(sm + OFF_V), 8192, 1024);
        const uint64_t dT1 = sw128_desc(smem_u32(sm + OFF_T1), 16, 1024);
        const uint64_t dT2 = sw128_desc(smem_u32(sm + OFF_T2), 16, 1024);
        const uint64_t dAS = sw128_desc(smem_u32(sm + OFF_AS), 16, 1024);
        const uint64_t dWT = sw128_desc(smem_u32(sm + OFF_WT), 8192, 1024);
        const uint64_t dAW = sw128_desc(smem_u32(sm + OFF_AW), 16, 1024);
        const uint64_t dAWD = sw128_desc(smem_u32(sm + OFF_AWD), 16, 1024);
        const uint64_t dP = sw128_desc(smem_u32(sm + OFF_P), 16, 1024);
        constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);
        constexpr uint32_t ID_MNK = idesc_bf16(128, 64, true, false);
        constexpr uint32_t ID_NEG = idesc_bf16(128, 64, false, true, true);
        constexpr uint32_t ID_S = idesc_bf16(128, DK, false, true);
        auto mma_p1 = [&](int c) {
            const uint64_t kq = dK16 + (uint64_t)((c & 1) * 32768 >> 4);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint64_t d = kq + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_bf16_ss(tb + TM_XP, d, d, ID_KK, kk > 0);
            }
            mma_commit(&bars[B_P1]);
        };
        auto mma_p2 = [&](int c) {
            const uint64_t kmn = dKmn + (uint64_t)((c & 1) * 32768 >> 4);
            const uint32_t x1 = TM_X1 + (uint32_t)(c & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tb + TM_XW, kmn + (uint64_t)(kk * 2048 >> 4), dT2 + (uint64_t)(kk * 32 >> 4), ID_MNK, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tb + x1, dV + (uint64_t)(kk * 2048 >> 4), dT1 + (uint64_t)(kk * 32 >> 4), ID_MNK, kk > 0);
            mma_commit(&bars[B_P2]);
        };
        auto mma_p3 = [&](int c) {
            const uint64_t kq = dK16 + (uint64_t)(((c & 1) * 32768 + 8192) >> 4);
            const uint32_t x1 = TM_X1 + (uint32_t)(c & 1) * 64, x2 = TM_X2 + (uint32_t)(c & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk)
                mma_bf16_ss(tb + x1, dAS + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                            dWT + (uint64_t)(kk * 2048 >> 4), ID_NEG, 1);
            mma_commit(&bars[B_P3]);        // the chain waits for Wt^T only
            if (!write_o) return;           // phase A: no output products
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_bf16_ss(tb + x2, dAS + off, kq + off, ID_KK, kk > 0);
            }
        };
        auto mma_p4 = [&](int c) {
            const uint64_t kmn = dKmn + (uint64_t)((c & 1) * 32768 >> 4);
            const uint64_t pp = dP + (uint64_t)((c & 1) * 8192 >> 4);
            const uint32_t x2 = TM_X2 + (uint32_t)(c & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tb + TM_S, dAWD + (uint64_t)(kk * 32 >> 4), kmn + (uint64_t)(kk * 2048 >> 4), ID_S, 1);
            if (write_o) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tb + x2, dAW + (uint64_t)(kk * 32 >> 4), pp + (uint64_t)(kk * 32 >> 4), ID_KK, 1);
            }
            mma_commit(&bars[B_SDONE + (c & 1)]);
        };
        int n1 = 0, n2 = 0, n3 = 0, n4 = 0, nK = 0, nV = 0;      // actions issued
        load_kq(0); ++nK;
        if (nch > 1) { load_kq(1); ++nK; }
        load_v(0); ++nV;
        if (W(B_KFULL, 0)) { tc_fence_after(); mma_p1(0); ++n1; }
        if (W(B_TREADY, 0) && W(B_VFULL, 0)) { tc_fence_after(); mma_p2(0); ++n2; }
        if (nch > 1 && W(B_KFULL + 1, 0)) { tc_fence_after(); mma_p1(1); ++n1; }
        for (int c = 0; c < nch && ok; ++c) {
            if (W(B_AS, c) && W(B_WQ, c) && (c < 2 || W(B_X2FREE + (c & 1), (c - 2) >> 1))) {
                tc_fence_after(); mma_p3(c); ++n3;
            }
            if (W(B_AW, c)) { tc_fence_after(); mma_p4(c); ++n4; }
            if (c + 2 < nch && W(B_SDONE + (c & 1), c >> 1)) { load_kq(c + 2); ++nK; }
            if (c + 1 < nch && W(B_P2, c)) { load_v(c + 1); ++nV; }
            if (c + 1 < nch && W(B_TREADY, c + 1) && W(B_VFULL, c + 1) &&
                (c < 1 || W(B_X1FREE + ((c - 1) & 1), (c - 1) >> 1))) {
                tc_fence_after(); mma_p2(c + 1); ++n2;
            }
            if (c + 2 < nch && W(B_KFULL + (c & 1), (c + 2) >> 1)) { tc_fence_after(); mma_p1(c + 2); ++n1; }
        }
        // drain: every issued commit group and load completes before TMEM is freed
        if (!ok) {
            *abort_flag = 1;
            if (n1 > 0) mbar_wait(&bars[B_P1], (n1 - 1) & 1);
            if (n2 > 0) mbar_wait(&bars[B_P2], (n2 - 1) & 1);
            if (n3 > 0) mbar_wait(&bars[B_P3], (n3 - 1) & 1);
            if (n4 > 0) mbar_wait(&bars[B_SDONE + ((n4 - 1) & 1)], ((n4 - 1) >> 1) & 1);
            if (nK > 0) mbar_wait(&bars[B_KFULL + ((nK - 1) & 1)], ((nK - 1) >> 1) & 1);
            if (nV > 0) mbar_wait(&bars[B_VFULL], (nV - 1) & 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tb, TM_COLS);
}

}  // namespace pfws
}  // namespace jet
