// K2a: state-independent preparation of every chunk of the chunked Gated
// DeltaNet prefill (Jet-Nemotron paper, section 2.3, gated delta rule in
// chunked WY / UT form), one CTA per (sequence, head, chunk), all at once.
//
// Everything in a chunk that does not depend on the running state is a
// function of that chunk's q, k, g and b alone, so it is computed here in
// parallel over all chunks and written to a per-chunk "image" in global
// memory; the chain kernel (K2b) then only runs the state products. The image
// holds bf16 operand tiles in the 128-byte swizzled layout the tensor cores
// read (so the chain kernel copies them into shared memory unchanged) and a
// few float vectors:
//   T1   [64 r][64 i]    T diag(b)                       (U^T = V^T T1^T)
//   W^T  [dk j][64 r]    (T diag(b gam / |k|) K)^T         (Wt^T = U^T - S W^T)
//   vec  dik[64] = d_i / |k_i|, then gam_{L-1}
//   P    [64 r][64 i]    exp(G_r - G_i) q^_r.k^_i (i <= r) (outputs only)
//   Q~   [64 r][dk]      diag(gam / |q|) Q, 64-column blocks (outputs only)
// T1, W^T and vec come first, so a pass without outputs copies a prefix.
//
// Flow of one CTA (256 threads, named barrier 1 = the whole CTA): TMA of the
// K / Q tile; P1 = [K; Q] K^T on tcgen05 while the per-token vectors are
// formed; A and P; the UT inverse; T1 / T2; P2b = K^T T2^T on tcgen05 while
// Q~ is formed; W^T. Tiles are staged in shared memory and written with bulk
// copies.
#pragma once
#include "k_prefill_common.cuh"

namespace jet {
namespace pfws {

constexpr int PREP_THREADS = 256;

// per-chunk image layout (bytes; every tile 1024-aligned)
template <int DK>
struct Img {
    static constexpr int NKB = (DK + 63) / 64;
    static constexpr uint32_t T1 = 0;
    static constexpr uint32_t WT = 8192;
    static constexpr uint32_t VEC = WT + DK * 128;
    static constexpr uint32_t A_BYTES = VEC + 1024;     // prefix used without outputs
    static constexpr uint32_t P = A_BYTES;
    static constexpr uint32_t Q = P + 8192;
    static constexpr uint32_t BYTES = Q + NKB * 8192;
    static_assert(WT % 1024 == 0 && VEC % 1024 == 0 && P % 1024 == 0 && Q % 1024 == 0, "image alignment");
};

// shared memory of the preparation kernel (bytes from a 1024-aligned base)
template <int DK>
struct PrepSmem {
    static constexpr int NKB = (DK + 63) / 64;
    static constexpr uint32_t KQ = 0;                              // per 64-col block [K 8K | Q 8K]
    static constexpr uint32_t T2 = KQ + NKB * 16384;
    static constexpr uint32_t T1 = T2 + 8192;                      // staging of the image tiles
    static constexpr uint32_t P = T1 + 8192;
    static constexpr uint32_t WT = P + 8192;
    static constexpr uint32_t AF = WT + ((DK * 128 + 1023) / 1024) * 1024;
    static constexpr uint32_t XS = AF + AF_BYTES;
    static constexpr uint32_t VEC = XS + XS_BYTES;                 // 8 x 64 fp32
    static constexpr uint32_t PN = VEC + 2048;
    static constexpr uint32_t IV = PN + 1024;                      // vec image staging
    static constexpr uint32_t BAR = IV + 1024;
    static constexpr uint32_t TSLOT = BAR + 64;
    static constexpr uint32_t BYTES = TSLOT + 16 + 1024;           // + alignment slack
    static_assert(2 * BYTES <= 232448, "two CTAs per SM");
};

template <int DK>
__global__ void __launch_bounds__(PREP_THREADS, 2)
gdn_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const float* __restrict__ g, const float* __restrict__ beta, uint8_t* __restrict__ img,
                      int Tn, int H) {
    using SM = PrepSmem<DK>;
    using IM = Img<DK>;
    constexpr int NKB = SM::NKB;
    constexpr int KSTEPS = DK / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::BAR);     // 0: K/Q landed, 1: P1, 2: P2b
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + SM::TSLOT);
    const int tid = threadIdx.x;
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nct = gridDim.x;
    const int t0 = c * C, L = min(C, Tn - t0);
    const int z = (int)((long long)b * Tn + t0);
    uint8_t* out = img + (((size_t)b * H + h) * nct + c) * IM::BYTES;
    constexpr uint32_t TM_XP = 0, TM_XW = 64;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
    }
    if (tid < 32) tmem_alloc(tslot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tslot;
    if (tid == 0) {
        mbar_expect_tx(&bars[0], (uint32_t)(NKB * 16384));
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
            tma_load_3d(sm + SM::KQ + kb * 16384, &tm_k, &bars[0], kb * 64, h, z);
            tma_load_3d(sm + SM::KQ + kb * 16384 + 8192, &tm_q, &bars[0], kb * 64, h, z);
        }
    }
    float gb = 0.f;
    if (tid < 128 && (tid & 63) < L) {
        const long long off = ((long long)z + (tid & 63)) * H + h;
        gb = tid < 64 ? g[off] : beta[off];
    }
    Vec V = vec_from(reinterpret_cast<float*>(sm + SM::VEC));
    float* AF = reinterpret_cast<float*>(sm + SM::AF);
    float* XS = reinterpret_cast<float*>(sm + SM::XS);
    float* PN = reinterpret_cast<float*>(sm + SM::PN);
    float* IV = reinterpret_cast<float*>(sm + SM::IV);
    const uint64_t dK16 = sw128_desc(smem_u32(sm + SM::KQ), 16, 1024);       // [K; Q] K-major
    const uint64_t dKmn = sw128_desc(smem_u32(sm + SM::KQ), 16384, 1024);    // K as MN-major
    const uint64_t dT2 = sw128_desc(smem_u32(sm + SM::T2), 16, 1024);
    constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_MNK = idesc_bf16(128, 64, true, false);

    bool issued1 = false, issued2 = false;           // MMA groups in flight (thread 0)
    bool ok = mbar_wait(&bars[0], 0);
    if ((ok = __syncthreads_and(ok))) {
        if (tid == 0) {   // P1: [K; Q] K^T -> XP
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint64_t d = dK16 + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_bf16_ss(tb + TM_XP, d, d, ID_KK, kk > 0);
            }
            mma_commit(&bars[1]);
            issued1 = true;
        }
        prep_vectors<DK>(sm + SM::KQ, V, PN, gb, L, tid, 1);
        ok = mbar_wait(&bars[1], 0);
    }
    if ((ok = __syncthreads_and(ok))) {
        tc_fence_after();
        prep_e1(tb + TM_XP, V, AF, sm + SM::P, tid);
        named_sync(1, PREP_THREADS);
        ut_inverse(AF, XS, tid, 1);
        prep_t1t2(AF, V, sm + SM::T1, sm + SM::T2, tid);
        if (tid < 64) IV[tid] = V.dcy[tid] * V.ik[tid];
        else if (tid == 64) IV[64] = V.gam[L - 1];
        fence_async_smem();
        tc_fence_before();
        named_sync(1, PREP_THREADS);
        if (tid == 0) {   // P2b: K^T T2^T -> XW; the finished tiles go out
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tb + TM_XW, dKmn + (uint64_t)(kk * 2048 >> 4), dT2 + (uint64_t)(kk * 32 >> 4), ID_MNK,
                            kk > 0);
            mma_commit(&bars[2]);
            issued2 = true;
            bulk_store(out + IM::T1, sm + SM::T1, 8192);
            bulk_store(out + IM::VEC, sm + SM::IV, 1024);
            bulk_store(out + IM::P, sm + SM::P, 8192);
            bulk_commit();
        }
        prep_qtilde<DK>(sm + SM::KQ, V, tid);           // P1 has read Q; P2b reads only K
        fence_async_smem();
        named_sync(1, PREP_THREADS);
        if (tid == 0) {
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) bulk_store(out + IM::Q + kb * 8192, sm + SM::KQ + kb * 16384 + 8192, 8192);
            bulk_commit();
        }
        ok = mbar_wait(&bars[2], 0);
        if ((ok = __syncthreads_and(ok))) {
            tc_fence_after();
            prep_wt<DK>(tb + TM_XW, sm + SM::WT, tid);
            fence_async_smem();
            named_sync(1, PREP_THREADS);
            if (tid == 0) {
                bulk_store(out + IM::WT, sm + SM::WT, DK * 128);
                bulk_commit();
            }
        }
    }
    if (tid == 0) {
        bulk_wait_all();             // shared memory stays valid until the copies have read it
        if (!ok) {                   // a wait ran out: let issued loads / MMAs finish (bounded)
            mbar_wait(&bars[0], 0);
            if (issued1) mbar_wait(&bars[1], 0);
            if (issued2) mbar_wait(&bars[2], 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid < 32) tmem_dealloc(tb, 128);
}

}  // namespace pfws
}  // namespace jet
