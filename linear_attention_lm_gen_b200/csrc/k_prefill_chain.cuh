// K2b: the state chain of the chunked Gated DeltaNet prefill (Jet-Nemotron
// paper, section 2.3), fed by the per-chunk images of K2a.
//
// With T1, W^T, P, Q~ and the decay vectors of every chunk already in global
// memory, what remains per chunk is the part that depends on the state
// (same notation as the preparation kernel):
//   U^T  = V^T T1^T                    P2a  (state-independent, runs ahead)
//   Wt^T = U^T - S W^T                 P3
//   O^T  = S Q~^T + Wt^T P^T           P5a / P5b (output products)
//   S   <- gam_{L-1} S + Wt^T diag(d/|k|) K   (E4 scales S in TMEM, then P4)
// One CTA = (sequence, head, 128 state rows) of one segment; the float32
// state lives in TMEM, its bf16 copy is the A operand of P3 / P5a.
//
//   warps 0-3  CHAIN  E4: S -> bf16 copy and S <- gam_L S;  E5: Wt^T -> bf16
//                     (plain and scaled by d/|k|); after each of them the
//                     group's first thread issues the state product itself
//                     (P3 after E4, P4 after E5), so no handoff to another
//                     thread sits on the chain
//   warps 4-7  OUT    E6: O^T (TMEM) -> staging -> global, off the chain
//   warp 10    LOAD   one thread issues the bulk copies of the images, the TMA
//                     loads of K and V as soon as their buffers are free, and
//                     the products off the chain: P2a (U^T, state-independent,
//                     one chunk ahead), P5a and P5b (outputs). They are issued
//                     into the chain's conversion windows, where the tensor
//                     pipe has nothing of the chain's: P5a(c) and P2a(c+1) once
//                     P3(c) has completed (they run during E5(c)), P5b(c) once
//                     P4(c) has completed (it runs during E4(c+1)), so they
//                     never queue in front of a state product. P5a and P5b
//                     complete on barriers of their own: the next chunk's E4
//                     waits only for P5a (which reads the bf16 S copy), its E5
//                     only for P5b (which reads Wt^T)
//   (warps 8 and 9 have no role: the load thread sits on the scheduler of
//   warp 2, away from the group pollers of warps 0 and 4)
//
// Buffers: images double-buffered (the copy of chunk c+2 starts once chunk c
// is finished), V double-buffered (V(c+2) once P2a(c) is done), K
// double-buffered for dk <= 96 (K(c+2) once P4(c) is done) and single for
// dk = 128 (K(c+1) once P4(c) is done; shared memory is full); outputs are
// staged 32 tokens at a time, or 16 where the images leave less room (dk = 96).
// TMEM: S, X1[2] (U^T then Wt^T), X2[2] (O^T) =
// 384 of 512 columns. The roles on the critical path (chain warps, MMA
// thread) spin on the mbarrier before they start to sleep between polls, so
// they wake within tens of cycles; the others sleep between polls and leave
// the issue slots to them.
//
// Segments (sequence parallelism, one pass). The recurrence is affine in the
// state, so with P segments every segment runs at once: segment 0 from S0,
// the others from a zero state, each writing provisional outputs O0 and its
// end state E_p. For p >= 1 an extra "transition" slice starts from the
// identity with zero values; its state is the product Phi_c of the per-token
// transitions since the segment start, and its output products give
//   Qe_c = (Q~ - P W) Phi_c^T      (64 tokens x dk, written per chunk)
// which is exactly what the start state multiplies in the outputs:
//   O_c = O0_c + Qe_c S*^T,  S* = the segment's true start state.
// The segment combine then chains S*_{p+1} = S*_p A_p + E_p (A_p = Phi at the
// segment end) and a correction kernel adds Qe_c S*^T to the outputs.
//
// CONV: the V tiles hold the raw values and the images were prepared with
// the dynamic causal conv (Jet-Nemotron paper, section 2.4) folded into T1:
// U^T = V^T M^T + Vh^T MH, where Vh = the 16 tokens before the chunk (only the
// last three have non-zero weights). Vh is the tail of the previous chunk's V
// tile, still in shared memory: V(c+1) is loaded once P2a(c) is done (one
// chunk ahead instead of two), and the tail before a segment's first chunk
// is loaded on its own (from V, or from the history at a sequence start).
// So v' is never formed at all; the last segment writes the new history (the
// last three raw values) from global memory.
#pragma once
#include "k_prefill_chunkprep.cuh"

namespace jet {
namespace pfch {

using namespace pfws;

constexpr int NCH_T = 128, NOUT = 128;
constexpr int THREADS = NCH_T + NOUT + 96;            // 352
constexpr int OUT0 = NCH_T, LOAD0 = NCH_T + NOUT + 64;   // warp 10

// bounded wait: spin on the phase first, then poll with short sleeps; gives up
// (error word + CTA abort flag) when the wait time limit runs out or another
// thread raised the abort flag
__device__ __forceinline__ bool wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    for (uint32_t i = 0; i < 2048; ++i)
        if (mbar_test_wait(bar, parity)) return true;
    return wait_bar(bar, parity, abort_flag);
}
// A group waits for one mbarrier phase: its first thread polls (spinning when
// `spin`), the others wait at the group's named barrier, which costs no issue
// slots and keeps the shared-memory pipe free for the MMA-issuing thread.
// True on every thread of the group iff the wait succeeded.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int bid, int n,
                                           bool poller, bool spin) {
    bool ok = true;
    if (poller) ok = spin ? wait_spin(bar, parity, abort_flag) : wait_bar(bar, parity, abort_flag);
    return group_all(bid, n, ok);
}

template <int DK>
struct ChainSmem {
    static constexpr int NKB = (DK + 63) / 64;
    static constexpr int NKBUF = DK <= 96 ? 2 : 1;           // K tiles in flight
    static constexpr uint32_t IB = ((Img<DK>::BYTES + 1023) / 1024) * 1024;
    static constexpr uint32_t IMG = 0;                       // [2] images
    static constexpr uint32_t K = IMG + 2 * IB;              // [NKBUF] x NKB x [64 tok][64 feat]
    static constexpr uint32_t V = K + NKBUF * NKB * 8192;    // [2] x 2 x [64 tok][64 ch]
    static constexpr uint32_t AS = V + 2 * 16384;            // NKB x [128 rows][64 feat] bf16 S
    static constexpr uint32_t AW = AS + NKB * 16384;         // Wt^T
    static constexpr uint32_t AWD = AW + 16384;              // Wt^T diag(d/|k|)
    static constexpr uint32_t OUT = AWD + 16384;             // [OUT_TOK tok][128 ch] bf16 output staging
    static constexpr int OUT_TOK = OUT + 8192 + 256 + 32 <= 232448 ? 32 : 16;
    static constexpr uint32_t BAR = OUT + OUT_TOK * 256;
    static constexpr uint32_t TSLOT = BAR + 256;
    static constexpr uint32_t ABORT = TSLOT + 16;
    // no alignment slack: the kernel checks that dynamic shared memory starts
    // on a 1024-byte boundary (the swizzled tiles need it) and flags an error
    // instead of running otherwise
    static constexpr uint32_t BYTES = ABORT + 16;
    static_assert(BYTES <= 232448, "shared memory budget");
};

constexpr uint32_t TM_S = 0, TM_X1 = 128, TM_X2 = 256, TM_COLS = 512;

// raw-V conv inputs of the CONV instantiation
struct ChainConv {
    const __nv_bfloat16* v;          // raw v [B*T][H][dv] (the tensor map's tensor)
    const __nv_bfloat16* hist_in;    // [B][3][H][dv] raw v_{-3..-1}, or null (zeros)
    __nv_bfloat16* hist_out;         // [B][3][H][dv] last three raw tokens, or null
};

#ifdef JET_TEST_WAIT_EXPIRY
// Test builds only (never in the library): while set, the load thread leaves
// out P2a of chunk 1, so the chain's bounded wait for it runs out and the
// kernel winds down with JET_ERR_TIMEOUT.
__device__ int g_test_skip_p2a = 0;
#endif

// one pass over all segments (see the header comment); P = 1 is the plain pass
struct ChainSeg {
    int nseg;                 // P
    int seg_chunks;           // chunks per segment (the last may be shorter)
    float* Eo;                // P > 1: end states [B][P][H][dv][dk] (segment 0 from S0, the others from 0)
    float* Ao;                // P > 1: transitions [B][P][H][dk][a_ld] (p >= 1)
    __nv_bfloat16* Qe;        // P > 1: output corrections [B][H][nct][64][dk] (chunks of segments p >= 1)
    int a_ld;                 // row stride of Ao (floats)
    int trans0;               // range mode (P = 1): segment 0 has a transition slice too, writing Ao and Qe
};

enum {
    B_IMG = 0,        // [2] image landed
    B_K = 2,          // [NKBUF] K tile landed
    B_V = 4,          // [2] V tile landed
    B_P2 = 6,         // [2] P2a complete (per V buffer, so no waiter lags two phases)
    B_P3 = 8,         // P3 complete
    B_SDONE = 9,      // [2] P4 complete
    B_P5A = 11,       // [2] P5a complete (the bf16 S copy free)
    B_X2FREE = 13,    // [2] O^T read (out)
    B_ODONE = 15,     // [2] P5b complete (O^T ready, Wt^T free)
    B_H0 = 17,        // the values before a segment's first chunk landed (CONV)
    NBARS = 18
};

// tm_vh / tm_hh (CONV): 16-row boxes of V ([B*T][H][dv]) and of the history
// ([B*3][H][dv]; tm_vh again without one) for the values before a segment
template <int DK, bool CONV>
__global__ void __launch_bounds__(THREADS, 1)
gdn_prefill_chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_vh, const __grid_constant__ CUtensorMap tm_hh,
                         const uint8_t* __restrict__ img, const float* S0, __nv_bfloat16* __restrict__ o,
                         float* S_out, int Tn, int H, int dv, const ChainSeg seg, const ChainConv cv,
                         const __grid_constant__ SeqMap sq) {
    static_assert(DK % 32 == 0 && DK >= 64 && DK <= 128, "DK in {64, 96, 128}");
    using SM = ChainSmem<DK>;
    using IM = Img<DK>;
    constexpr int NKB = SM::NKB;
    constexpr int KSTEPS = DK / 16;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::BAR);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + SM::TSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + SM::ABORT);

    const int tid = threadIdx.x, warp = tid >> 5;
    if (smem_u32(sm) & 1023u) {                           // whole CTA, before any barrier
        if (tid == 0) flag_error(DEVERR_DATA);
        return;
    }
    const int ns = dv / ROWS;
    // this CTA's sequence b and its segment p_seg of P (gs: global segment index),
    // the sequence's tokens Tb starting at row tok0, its chunks at nctH0 + h nct_b
    const int h = blockIdx.y, gs = blockIdx.z;
    int b, p_seg, P, Tb, tok0, nct, nctH0, segc;
    if (sq.nseq == 0) {
        P = seg.nseg;
        b = gs / P;
        p_seg = gs % P;
        Tb = Tn;
        tok0 = b * Tn;
        nct = (Tn + C - 1) / C;
        nctH0 = b * H * nct;
        segc = seg.seg_chunks;
    } else {
        b = seq_of(sq.seg, sq.nseq, gs, 1);
        p_seg = gs - sq.seg[b];
        P = sq.seg[b + 1] - sq.seg[b];
        tok0 = sq.tok[b];
        Tb = sq.tok[b + 1] - tok0;
        nct = sq.chunk[b + 1] - sq.chunk[b];
        nctH0 = sq.chunk[b] * H;
        segc = sq.seg_chunks;
    }
    const bool trans = blockIdx.x == ns;                  // transition slice (p >= 1)
    if (trans && p_seg == 0 && !seg.trans0) return;      // whole CTA, before any barrier
    const int c0 = blockIdx.x * ROWS;                     // transition slice: past dv, V reads as zero
    const long long bh = (long long)b * H + h;
    const int cbeg = p_seg * segc;
    const int tbeg = cbeg * C;
    const int tend = min(Tb, tbeg + segc * C);
    const int nch = (tend - tbeg + C - 1) / C;
    constexpr bool write_o = true;                        // every slice has output products (trans: Qe)
    const long long img0 = (long long)nctH0 + (long long)h * nct;   // image / Qe index of the sequence's chunk 0
    const uint8_t* img_bh = img + (size_t)img0 * IM::BYTES;
    auto img_at = [&](int c) -> const uint8_t* { return sm + SM::IMG + (uint32_t)(c & 1) * SM::IB; };

    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (tid == LOAD0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (CONV) {
            tma_prefetch_desc(&tm_vh);
            tma_prefetch_desc(&tm_hh);
        }
    }
    if (warp == 0) tmem_alloc(tslot, TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tslot;
    pdl_wait();                                           // images, S0, K and V are read from here on
    pdl_trigger();

    const uint64_t dAS = sw128_desc(smem_u32(sm + SM::AS), 16, 1024);
    auto as_off = [&](int kk) { return (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4); };
    auto ioff = [&](int c, uint32_t off) { return (uint64_t)((((uint32_t)(c & 1) * SM::IB) + off) >> 4); };

    if (warp < 4) {
        // =============================================================== CHAIN
        const int ct = tid;
        constexpr int NKBUF = SM::NKBUF;
        const uint64_t dImgMN = sw128_desc(smem_u32(sm + SM::IMG), 8192, 1024);   // W^T (MN-major)
        const uint64_t dKmn = sw128_desc(smem_u32(sm + SM::K), 8192, 1024);       // K as MN-major
        const uint64_t dAWD = sw128_desc(smem_u32(sm + SM::AWD), 16, 1024);
        constexpr uint32_t ID_NEG = idesc_bf16(128, 64, false, true, true);
        constexpr uint32_t ID_S = idesc_bf16(128, DK, false, true);
        int n3 = 0, n4 = 0;                                  // commit groups issued (thread 0)
        bool live = true;                                    // thread 0: every wait so far succeeded
        const uint32_t lb = (uint32_t)(warp * 32) << 16;
        {   // initial state (row ct of the slice)
            const float* src = (p_seg == 0 && !trans && S0) ? S0 + (bh * dv + c0 + ct) * DK : nullptr;
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
        for (int c = 0; c < nch; ++c) {
            const int p = c & 1;
            const float* iv = reinterpret_cast<const float*>(img_at(c) + IM::VEC);   // dik[64], gam_{L-1}
            bool okw = true;
            if (ct == 0) {
                // S updated (P4), the bf16 S copy no longer read (P5a), image landed
                okw = live && (c < 1 || wait_spin(&bars[B_SDONE + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag));
                okw = okw && (c < 1 || !write_o ||
                              wait_spin(&bars[B_P5A + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag));
                okw = okw && wait_spin(&bars[B_IMG + p], (c >> 1) & 1, abort_flag);
            }
            if (!group_all(2, NCH_T, okw)) break;
            tc_fence_after();
            // ---- E4: S -> bf16 copy, S <- gam_L S
            {   // 64 columns (one SW128 block of the copy) per TMEM load wait (32 at dk = 128: registers)
                const float gL = iv[64];
                constexpr int NB = DK <= 96 ? 2 : 1;
#pragma unroll
                for (int c2 = 0; c2 < DK / 32; c2 += NB) {
                    const int nb = min(NB, DK / 32 - c2);
                    uint32_t x[NB][32];
#pragma unroll
                    for (int u = 0; u < NB; ++u)
                        if (u < nb) tmem_ld32(tb + lb + TM_S + (c2 + u) * 32, x[u]);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < NB; ++u) {
                        if (u >= nb) break;
                        const int cb = c2 + u;
                        uint8_t* tile = sm + SM::AS + (cb >> 1) * 16384;
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            float f[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(x[u][8 * ch + e]);
                            *reinterpret_cast<uint4*>(tile + sw128_off(ct, ((cb & 1) * 32 + ch * 8) * 2)) = pack8(f);
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) x[u][j] = __float_as_uint(gL * __uint_as_float(x[u][j]));
                        tmem_st32(tb + lb + TM_S + (c2 + u) * 32, x[u]);
                    }
                }
                tmem_st_wait();
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NCH_T);
            // ---- P3 (thread 0): X1[c&1] -= S W^T  (= Wt^T), once U^T of the chunk is in X1
            bool okp = true;
            if (ct == 0) {
                okp = wait_spin(&bars[B_P2 + (c & 1)], (c >> 1) & 1, abort_flag);
                if (okp) {
                    tc_fence_after();
                    const uint32_t x1 = TM_X1 + (uint32_t)(c & 1) * 64;
#pragma unroll
                    for (int kk = 0; kk < KSTEPS; ++kk)
                        mma_bf16_ss(tb + x1, dAS + as_off(kk), dImgMN + ioff(c, IM::WT + kk * 2048), ID_NEG, 1);
                    mma_commit(&bars[B_P3]);
                    ++n3;
                    okp = wait_spin(&bars[B_P3], c & 1, abort_flag);
                }
                // E5 overwrites Wt^T: the previous chunk's P5b has read it
                okp = okp && (c < 1 || !write_o ||
                              wait_spin(&bars[B_ODONE + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag));
                live = okp;
            }
            // ---- E5: Wt^T -> bf16 (plain and scaled by d/|k|)
            if (!group_all(2, NCH_T, okp)) break;
            tc_fence_after();
            {
                const uint32_t x1 = TM_X1 + (uint32_t)p * 64;
                uint32_t xx[2][32];
                tmem_ld32(tb + lb + x1, xx[0]);
                tmem_ld32(tb + lb + x1 + 32, xx[1]);
                tmem_ld_wait();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t* x = xx[half];
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float f[8], fd[8];
                        const float4 d0 = *reinterpret_cast<const float4*>(iv + half * 32 + ch * 8);
                        const float4 d1 = *reinterpret_cast<const float4*>(iv + half * 32 + ch * 8 + 4);
                        const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            f[e] = __uint_as_float(x[ch * 8 + e]);
                            fd[e] = f[e] * dd[e];
                        }
                        const uint32_t off = sw128_off(ct, (half * 32 + ch * 8) * 2);
                        *reinterpret_cast<uint4*>(sm + SM::AW + off) = pack8(f);
                        *reinterpret_cast<uint4*>(sm + SM::AWD + off) = pack8(fd);
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            named_sync(2, NCH_T);
            // ---- P4 (thread 0): S += Wt^T diag(d/|k|) K, once the K tile is in
            if (ct == 0) {
                live = wait_spin(&bars[B_K + c % NKBUF], (c / NKBUF) & 1, abort_flag);
                if (live) {
                    tc_fence_after();
                    const uint64_t dk_ = dKmn + (uint64_t)(((uint32_t)(c % NKBUF) * NKB * 8192) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tb + TM_S, dAWD + (uint64_t)(kk * 32 >> 4), dk_ + (uint64_t)(kk * 2048 >> 4), ID_S, 1);
                    mma_commit(&bars[B_SDONE + (c & 1)]);
                    ++n4;
                }
            }
        }
        // final state of the segment (after the last P4)
        bool fin = true;
        if (ct == 0)
            fin = live && !*abort_flag && nch > 0 && n4 == nch &&
                  wait_spin(&bars[B_SDONE + ((nch - 1) & 1)], ((nch - 1) >> 1) & 1, abort_flag);
        if (group_all(2, NCH_T, fin)) {
            tc_fence_after();
            float* dst = nullptr;
            if (trans) {                                      // the transition (p >= 1, or range mode)
                if (ct < DK) dst = seg.Ao + (((long long)gs * H + h) * DK + ct) * seg.a_ld;
            } else if (P == 1) {
                dst = S_out + (bh * dv + c0 + ct) * DK;
            } else {
                dst = seg.Eo + (((long long)gs * H + h) * dv + c0 + ct) * DK;
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
        if (ct == 0) {
            // every chain MMA this thread issued has completed before TMEM is freed
            // (immediate unless a wait ran out)
            if (!fin) *abort_flag = 1;
            if (n3 > 0) mbar_wait(&bars[B_P3], (n3 - 1) & 1);
            for (int j = max(0, n4 - 2); j < n4; ++j) mbar_wait(&bars[B_SDONE + (j & 1)], (j >> 1) & 1);
        }
    } else if (warp < 8) {
        // =============================================================== OUT
        constexpr int OUT_TOK = SM::OUT_TOK;                 // tokens per staging round
        const int ot = tid - OUT0;                           // channel of the slice
        const uint32_t lb = (uint32_t)((warp & 3) * 32) << 16;
        __nv_bfloat16* st = reinterpret_cast<__nv_bfloat16*>(sm + SM::OUT);
        const long long tstride = (long long)H * dv;
        bool run = true;
        for (int c = 0; c < nch && write_o; ++c) {
            if (!group_wait(&bars[B_ODONE + (c & 1)], (c >> 1) & 1, abort_flag, 3, NOUT, ot == 0, false)) {
                run = false;
                break;
            }
            tc_fence_after();
            const uint32_t x2 = TM_X2 + (uint32_t)(c & 1) * 64;
            const int t0 = tbeg + c * C, L = min(C, tend - t0);
            // value slices: o rows of this chunk; transition slice: Qe of the chunk
            // ([64 tokens][dk], rows of the slice = key features, only the first dk exist)
            __nv_bfloat16* obase = trans ? seg.Qe + ((size_t)img0 + cbeg + c) * C * DK
                                         : o + ((long long)tok0 + t0) * tstride + (long long)h * dv + c0;
            const long long rstride = trans ? (long long)DK : tstride;
            const int nchunk16 = trans ? DK / 8 : 16;
#pragma unroll
            for (int half = 0; half < 2; ++half) {           // 32 tokens from TMEM at a time
                uint32_t x[32];
                tmem_ld32(tb + lb + x2 + half * 32, x);
                tmem_ld_wait();
#pragma unroll
                for (int sub = 0; sub < 32 / OUT_TOK; ++sub) {
#pragma unroll
                    for (int j = 0; j < OUT_TOK; ++j)
                        st[j * ROWS + ot] = __float2bfloat16_rn(__uint_as_float(x[sub * OUT_TOK + j]));
                    if (half == 1 && sub == 0) tc_fence_before();
                    named_sync(3, NOUT);
                    if (half == 1 && sub == 0 && ot == 0) arrive(&bars[B_X2FREE + (c & 1)]);
#pragma unroll
                    for (int m = 0; m < OUT_TOK / 8; ++m) {  // OUT_TOK rows x 16 chunks of 16 bytes
                        const int qd = ot + m * NOUT, r = qd >> 4, cq = qd & 15;
                        const int tok = half * 32 + sub * OUT_TOK + r;
                        if (tok < L && cq < nchunk16)
                            *reinterpret_cast<uint4*>(obase + tok * rstride + cq * 8) =
                                *reinterpret_cast<const uint4*>(st + r * ROWS + cq * 8);
                    }
                    named_sync(3, NOUT);                     // staging free again
                }
            }
        }
        if (!run) *abort_flag = 1;
        // CONV: the new history, the last three raw values of the sequence (or of the old history)
        if (CONV && run && cv.hist_out && !trans && p_seg == P - 1 && c0 + ot < dv) {
            const int ch = c0 + ot;
#pragma unroll
            for (int k3 = 0; k3 < 3; ++k3) {
                const int tau = Tb - 3 + k3;
                __nv_bfloat16 val = __float2bfloat16_rn(0.f);
                if (tau >= 0) val = cv.v[((long long)tok0 + tau) * tstride + (long long)h * dv + ch];
                else if (cv.hist_in) val = cv.hist_in[((long long)b * 3 + 3 + tau) * tstride + (long long)h * dv + ch];
                cv.hist_out[((long long)b * 3 + k3) * tstride + (long long)h * dv + ch] = val;
            }
        }
    } else if (tid == LOAD0) {
        // =============================================================== LOAD
        // Two issuing threads, each in a fixed order (every awaited event
        // depends only on actions issued earlier in these orders or by the
        // other roles; a tcgen05 commit covers the issuing thread's MMAs):
        //   CHAIN thread 0: chunk c: P3(c) after E4(c) and P2a(c); P4(c) after
        //        E5(c) and K(c)
        //   LOAD (everything else): IMG(0) V(0) K(0) IMG(1) V(1) [K(1)] P2a(0);
        //        chunk c: V(c+2) (CONV: V(c+1)) after P2a(c); P5a(c) after P3(c)
        //        and X2[c&1] free; P2a(c+1) after IMG(c+1) and V(c+1); P5b(c)
        //        after P4(c); CONV: the segment's halo with V(0), before P2a(0);
        //        K(c+NKBUF) and IMG(c+2) after P5b(c)
        constexpr int NKBUF = SM::NKBUF;
        const uint64_t dImg = sw128_desc(smem_u32(sm + SM::IMG), 16, 1024);       // K-major tiles of the image
        bool ok = true;
        {
            // waits off the critical path sleep between polls
            auto WL = [&](int bar, int phase) {
                if (ok && !wait_bar(&bars[bar], (uint32_t)phase & 1u, abort_flag)) ok = false;
                return ok;
            };
            const uint32_t img_bytes = write_o ? IM::BYTES : IM::A_BYTES;
            auto zrow = [&](int c) { return tok0 + tbeg + c * C; };
            auto load_img = [&](int c) {
                uint64_t* bar = &bars[B_IMG + (c & 1)];
                mbar_expect_tx(bar, img_bytes);
                bulk_load(const_cast<uint8_t*>(img_at(c)), img_bh + (size_t)(cbeg + c) * IM::BYTES, img_bytes, bar);
            };
            auto load_k = [&](int c) {
                const int kb_ = c % NKBUF;
                uint64_t* bar = &bars[B_K + kb_];
                mbar_expect_tx(bar, (uint32_t)(NKB * 8192));
#pragma unroll
                for (int kb = 0; kb < NKB; ++kb)
                    tma_load_3d(sm + SM::K + (kb_ * NKB + kb) * 8192, &tm_k, bar, kb * 64, h, zrow(c));
            };
            auto load_v = [&](int c) {
                uint64_t* bar = &bars[B_V + (c & 1)];
                uint8_t* dst = sm + SM::V + (uint32_t)(c & 1) * 16384;
                mbar_expect_tx(bar, 16384);
                tma_load_3d(dst, &tm_v, bar, c0, h, zrow(c));
                tma_load_3d(dst + 8192, &tm_v, bar, c0 + 64, h, zrow(c));
            };
            // CONV: the 16 values before a segment's first chunk, into rows 48..63 of
            // V buffer 1 (where P2a(0) looks for the previous chunk's tail)
            auto load_h0 = [&]() {
                uint64_t* bar = &bars[B_H0];
                uint8_t* dst = sm + SM::V + 16384 + 48 * 128;
                mbar_expect_tx(bar, 2 * 16 * 128);
                // sequence start: the history's rows 0..2 at box rows 13..15, else all-zero rows
                // (coordinates below 0 read as zero; rows of other sequences only meet zero weights)
                const bool from_hist = tbeg == 0 && cv.hist_in != nullptr;
                const CUtensorMap* m = from_hist ? &tm_hh : &tm_vh;
                const int z = from_hist ? b * 3 - 13 : (tbeg == 0 ? -16 : tok0 + tbeg - 16);
                tma_load_3d(dst, m, bar, c0, h, z);
                tma_load_3d(dst + 8192, m, bar, c0 + 64, h, z);
            };
            const uint64_t dV = sw128_desc(smem_u32(sm + SM::V), 8192, 1024);
            const uint64_t dAW = sw128_desc(smem_u32(sm + SM::AW), 16, 1024);
            const uint64_t dImgMN = sw128_desc(smem_u32(sm + SM::IMG), 8192, 1024);   // MH (MN-major)
            constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);
            constexpr uint32_t ID_MNK = idesc_bf16(128, 64, true, false);
            constexpr uint32_t ID_MNMN = idesc_bf16(128, 64, true, true);
            auto mma_p2a = [&](int c) {      // X1[c&1] = V^T T1^T   (CONV: Vh^T MH + V^T M^T)
                const uint32_t x1 = TM_X1 + (uint32_t)(c & 1) * 64;
                const uint64_t dv_ = dV + (uint64_t)(((uint32_t)(c & 1) * 16384) >> 4);
                if (CONV) {   // the previous chunk's rows 48..63 (buffer (c-1)&1; c = 0: the segment's halo)
                    const uint64_t dvh = dV + (uint64_t)(((uint32_t)((c + 1) & 1) * 16384 + 48 * 128) >> 4);
                    mma_bf16_ss(tb + x1, dvh, dImgMN + ioff(c, IM::MH), ID_MNMN, 0);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tb + x1, dv_ + (uint64_t)(kk * 2048 >> 4), dImg + ioff(c, IM::T1 + kk * 32), ID_MNK,
                                CONV || kk > 0);
                mma_commit(&bars[B_P2 + (c & 1)]);
            };
            auto mma_p5a = [&](int c) {      // X2[c&1] = S Q~^T
                const uint32_t x2 = TM_X2 + (uint32_t)(c & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk)
                    mma_bf16_ss(tb + x2, dAS + as_off(kk), dImg + ioff(c, IM::Q + (kk >> 2) * 8192 + (kk & 3) * 32),
                                ID_KK, kk > 0);
                mma_commit(&bars[B_P5A + (c & 1)]);
            };
            auto mma_p5b = [&](int c) {      // X2[c&1] += Wt^T P^T
                const uint32_t x2 = TM_X2 + (uint32_t)(c & 1) * 64;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tb + x2, dAW + (uint64_t)(kk * 32 >> 4), dImg + ioff(c, IM::P + kk * 32), ID_KK, 1);
                mma_commit(&bars[B_ODONE + (c & 1)]);
            };
            int nK = 0, nV = 0, nI = 0, n2 = 0, n5a = 0, n5 = 0;   // loads / commit groups issued
            bool h0 = false;
            if (nch > 0) { load_img(0); ++nI; load_v(0); ++nV; load_k(0); ++nK; }
            if (CONV && nch > 0) { load_h0(); h0 = true; }
            if (nch > 1) { load_img(1); ++nI; }
            if (!CONV && nch > 1) { load_v(1); ++nV; }
            if (NKBUF == 2 && nch > 1) { load_k(1); ++nK; }
            if (nch > 0 && WL(B_IMG, 0) && WL(B_V, 0) && (!CONV || WL(B_H0, 0))) { tc_fence_after(); mma_p2a(0); ++n2; }
            for (int c = 0; c < nch && ok; ++c) {
                // the next V tile into the buffer P2a(c) has read (done early in chunk c):
                // V(c+2), or with CONV V(c+1) (its buffer held V(c-1), the halo of P2a(c))
                if (CONV && c + 1 < nch && WL(B_P2 + (c & 1), c >> 1)) { load_v(c + 1); ++nV; }
                if (!CONV && c + 2 < nch && WL(B_P2 + (c & 1), c >> 1)) { load_v(c + 2); ++nV; }
                // E5(c) window: P3(c) has completed (E4(c) wrote the S copy before it)
                if (WL(B_P3, c)) {
                    if (write_o && (c < 2 || WL(B_X2FREE + (c & 1), (c - 2) >> 1))) {
                        tc_fence_after(); mma_p5a(c); ++n5a;
                    }
                    if (c + 1 < nch && WL(B_IMG + ((c + 1) & 1), (c + 1) >> 1) &&
                        WL(B_V + ((c + 1) & 1), (c + 1) >> 1)) {
#ifdef JET_TEST_WAIT_EXPIRY
                        if (!(c == 0 && *reinterpret_cast<volatile int*>(&g_test_skip_p2a)))
#endif
                        { tc_fence_after(); mma_p2a(c + 1); ++n2; }
                    }
                }
                // E4(c+1) window: P4(c) has completed (E5(c) wrote Wt^T before it)
                if (WL(B_SDONE + (c & 1), c >> 1)) {
                    if (write_o) { tc_fence_after(); mma_p5b(c); ++n5; }
                    if ((c + NKBUF < nch || c + 2 < nch) && (!write_o || WL(B_ODONE + (c & 1), c >> 1))) {
                        if (c + NKBUF < nch) { load_k(c + NKBUF); ++nK; }
                        if (c + 2 < nch) { load_img(c + 2); ++nI; }
                    }
                }
            }
            // every issued load and commit group has completed before the CTA
            // frees its memory (the last one on each barrier; immediate unless
            // a wait ran out)
            if (!ok) *abort_flag = 1;
            for (int j = max(0, nK - NKBUF); j < nK; ++j) mbar_wait(&bars[B_K + j % NKBUF], (j / NKBUF) & 1);
            for (int j = max(0, nV - 2); j < nV; ++j) mbar_wait(&bars[B_V + (j & 1)], (j >> 1) & 1);
            for (int j = max(0, nI - 2); j < nI; ++j) mbar_wait(&bars[B_IMG + (j & 1)], (j >> 1) & 1);
            for (int j = max(0, n2 - 2); j < n2; ++j) mbar_wait(&bars[B_P2 + (j & 1)], (j >> 1) & 1);
            for (int j = max(0, n5a - 2); j < n5a; ++j) mbar_wait(&bars[B_P5A + (j & 1)], (j >> 1) & 1);
            for (int j = max(0, n5 - 2); j < n5; ++j) mbar_wait(&bars[B_ODONE + (j & 1)], (j >> 1) & 1);
            if (h0) mbar_wait(&bars[B_H0], 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tb, TM_COLS);
}

}  // namespace pfch
}  // namespace jet
