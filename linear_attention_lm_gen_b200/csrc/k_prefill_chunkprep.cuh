// K2a: state-independent preparation of every chunk of the chunked Gated
// DeltaNet prefill (Jet-Nemotron paper, section 2.3, gated delta rule in
// chunked WY / UT form), for all (sequence, head, chunk) items at once.
//
// Everything in a chunk that does not depend on the running state is a
// function of that chunk's q, k, g and b alone, so it is computed here in
// parallel over all chunks and written to a per-chunk "image" in global
// memory; the chain kernel (K2b) then only runs the state products. The image
// holds bf16 operand tiles in the 128-byte swizzled layout the tensor cores
// read (so the chain kernel copies them into shared memory unchanged) and a
// few float vectors:
//   T1   [64 r][64 i]    T diag(b)                       (U^T = V^T T1^T)
//                        or, with taps, M: T1 with the dynamic conv folded in
//   W^T  [dk j][64 r]    (T diag(b gam / |k|) K)^T         (Wt^T = U^T - S W^T)
//   vec  dik[64] = d_i / |k_i|, then gam_{L-1}
//   MH   [16 s][64 r]    with taps: the conv's reach into the previous
//                        chunk's last three raw values (see prep_mconv)
//   P    [64 r][64 i]    exp(G_r - G_i) q^_r.k^_i (i <= r) (outputs only)
//   Q~   [64 r][dk]      diag(gam / |q|) Q, 64-column blocks (outputs only)
// T1, W^T, vec and MH come first, so a pass without outputs copies a prefix.
//
// A CTA (256 threads, named barrier 1 = the whole CTA) walks items
// blockIdx.x, blockIdx.x + gridDim.x, ...; three CTAs share an SM, so three
// items are in flight per SM, and the K / Q tile of a CTA's next item is
// loaded (TMA) as soon as the current one has been consumed. Per item: P1 = [K; Q] K^T on
// tcgen05 while the per-token vectors are formed; A and P; the UT inverse;
// T1 / T2; P2b = K^T T2^T on tcgen05 while Q~ is formed; W^T. T1, P, W^T and
// the vectors are stored straight from registers (each warp store covers
// whole 128-byte rows or 16-byte pieces of them), Q~ by a bulk copy from
// its shared-memory tile.
#pragma once
#include "k_prefill_common.cuh"

namespace jet {
namespace pfws {

constexpr int PREP_THREADS = 256;
constexpr int PREP_KQBUF = 1;        // K / Q tiles in flight per CTA
constexpr int PREP_CTAS = 3;         // resident CTAs per SM (items in flight per SM)

// per-chunk image layout (bytes; every tile 1024-aligned)
template <int DK>
struct Img {
    static constexpr int NKB = (DK + 63) / 64;
    static constexpr uint32_t T1 = 0;
    static constexpr uint32_t WT = 8192;
    static constexpr uint32_t VEC = WT + DK * 128;
    static constexpr uint32_t MH = VEC + 1024;
    static constexpr uint32_t A_BYTES = MH + 2048;      // prefix used without outputs
    static constexpr uint32_t P = A_BYTES;
    static constexpr uint32_t Q = P + 8192;
    static constexpr uint32_t BYTES = Q + NKB * 8192;
    static_assert(WT % 1024 == 0 && VEC % 1024 == 0 && MH % 1024 == 0 && P % 1024 == 0 && Q % 1024 == 0,
                  "image alignment");
};

// shared memory of the preparation kernel (bytes from a 1024-aligned base)
template <int DK>
struct PrepSmem {
    static constexpr int NKB = (DK + 63) / 64;
    static constexpr uint32_t KQB = NKB * 16384;                   // one K / Q tile: [K 8K | Q 8K] per block
    static constexpr uint32_t KQ = 0;                              // [PREP_KQBUF] tiles
    static constexpr uint32_t T2 = KQ + PREP_KQBUF * KQB;
    static constexpr uint32_t AF = T2 + 8192;
    static constexpr uint32_t XS = AF + AF_BYTES;
    static constexpr uint32_t VEC = XS + XS_BYTES;                 // 8 x 64 fp32
    static constexpr uint32_t PN = VEC + 2048;
    static constexpr uint32_t TP = PN + 1024;                      // [2] taps of a chunk's tokens (see tp_slot)
    static constexpr uint32_t BAR = TP + 2 * TP_BYTES;
    static constexpr uint32_t TSLOT = BAR + 64;
    static constexpr uint32_t BYTES = TSLOT + 16 + 1024;           // + alignment slack
    static_assert(PREP_CTAS * (BYTES + 1024) <= 233472, "resident CTAs per SM");
};

// items = B * H * nct (dense) or H * (total chunks) (variable length), see
// item_info; the item index is also the image index. taps [tokens][H][4] or
// null: with taps the T1 slot holds M and MH is written (the chain then reads
// raw values); halo0: whether the values before each sequence's first token
// are a history (else MH of each sequence's first chunk is zero).
template <int DK>
__global__ void __launch_bounds__(PREP_THREADS, PREP_CTAS)
gdn_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const float* __restrict__ g, const float* __restrict__ beta, const float* __restrict__ taps,
                      int halo0, uint8_t* __restrict__ img, int Tn, int H, int nct, int n_items,
                      const __grid_constant__ SeqMap sq, int early) {
    using SM = PrepSmem<DK>;
    using IM = Img<DK>;
    constexpr int NKB = SM::NKB;
    constexpr int KSTEPS = DK / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + SM::BAR);     // 0, 1: K/Q landed; 2: P1; 3: P2b
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + SM::TSLOT);
    const int tid = threadIdx.x;
    constexpr uint32_t TM_XP = 0, TM_XW = 64;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
    }
    if (tid < 32) tmem_alloc(tslot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tslot;
    // The previous launch is waited for before the first global read, except
    // with `early`: then it is the same call's generator, which writes only the
    // taps, and everything else was complete before it began; q, k, g and beta
    // are read at once and the wait comes just before the first taps are.
    if (!early) pdl_wait();
    pdl_trigger();

    auto issue_load = [&](int item, int buf) {       // thread 0
        const ItemInfo it = item_info(item, Tn, H, nct, sq);
        uint8_t* dst = sm + SM::KQ + buf * SM::KQB;
        mbar_expect_tx(&bars[buf], (uint32_t)(NKB * 16384));
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
            tma_load_3d(dst + kb * 16384, &tm_k, &bars[buf], kb * 64, it.h, it.z);
            tma_load_3d(dst + kb * 16384 + 8192, &tm_q, &bars[buf], kb * 64, it.h, it.z);
        }
    };
    int nld[2] = {0, 0}, ndone[2] = {0, 0};          // loads issued / consumed per buffer (thread 0)
    int n1 = 0, n2 = 0;                               // MMA groups issued (thread 0)
    if (tid == 0)
        for (int j = 0; j < PREP_KQBUF; ++j)
            if (blockIdx.x + j * (int)gridDim.x < n_items) { issue_load(blockIdx.x + j * gridDim.x, j); ++nld[j]; }
    Vec V = vec_from(reinterpret_cast<float*>(sm + SM::VEC));
    float* AF = reinterpret_cast<float*>(sm + SM::AF);
    float* XS = reinterpret_cast<float*>(sm + SM::XS);
    float* PN = reinterpret_cast<float*>(sm + SM::PN);
    constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);
    constexpr uint32_t ID_MNK = idesc_bf16(128, 64, true, false);
    const uint64_t dT2 = sw128_desc(smem_u32(sm + SM::T2), 16, 1024);

    // g (tid < 64) or b (64 <= tid < 128) of one token of an item, 0 past the sequence end
    auto load_gb = [&](int item) -> float {
        if (item >= n_items || tid >= 128) return 0.f;
        const ItemInfo it = item_info(item, Tn, H, nct, sq);
        if ((tid & 63) >= it.L) return 0.f;
        const long long off = ((long long)it.z + (tid & 63)) * H + it.h;
        return tid < 64 ? g[off] : beta[off];
    };
    // taps of an item's tokens into TP[buf] (threads < 64; cp.async, zero past the sequence end)
    auto load_taps = [&](int item, int buf) {
        if (!taps || item >= n_items || tid >= 64) return;
        const ItemInfo it = item_info(item, Tn, H, nct, sq);
        const bool in = tid < it.L;
        const float* src = taps + (in ? ((long long)(it.z + tid) * H + it.h) * 4 : 0);
        const uint32_t dst = smem_u32(sm + SM::TP) + (uint32_t)buf * TP_BYTES + (uint32_t)tp_slot(tid) * 16u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(in ? 16u : 0u)
                     : "memory");
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    bool ok = true;
    int k = 0;
    if (!early) load_taps(blockIdx.x, 0);
    float gb_next = load_gb(blockIdx.x);
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
        const int buf = k % PREP_KQBUF;
        uint8_t* KQ = sm + SM::KQ + buf * SM::KQB;
        const ItemInfo info = item_info(item, Tn, H, nct, sq);
        const int L = info.L;
        uint8_t* out = img + (size_t)item * IM::BYTES;
        const float gb = gb_next;
        gb_next = load_gb(item + gridDim.x);            // in flight during this item
        if (!(ok = __syncthreads_and(mbar_wait(&bars[buf], (uint32_t)(k / PREP_KQBUF) & 1)))) break;
        if (tid == 0) {   // P1: [K; Q] K^T -> XP
            ++ndone[buf];
            tc_fence_after();
            const uint64_t dK16 = sw128_desc(smem_u32(KQ), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint64_t d = dK16 + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                mma_bf16_ss(tb + TM_XP, d, d, ID_KK, kk > 0);
            }
            mma_commit(&bars[2]);
            ++n1;
        }
        prep_vectors<DK>(KQ, V, PN, gb, L, tid, 1);
        if (early && k == 0) {                           // the generator's output from here on
            pdl_wait();
            load_taps(item, 0);
        }
        if (!(ok = __syncthreads_and(mbar_wait(&bars[2], (uint32_t)k & 1)))) break;
        tc_fence_after();
        prep_e1(tb + TM_XP, V, AF, out + IM::P, tid);
        if (taps && tid < 64) asm volatile("cp.async.wait_group 0;" ::: "memory");   // this item's taps (read by T1)
        named_sync(1, PREP_THREADS);
        ut_inverse(AF, XS, tid, 1);
        if (taps)
            prep_t1t2_conv(AF, V, reinterpret_cast<const float4*>(sm + SM::TP + (k & 1) * TP_BYTES), out + IM::T1,
                           out + IM::MH, sm + SM::T2, halo0 || info.c != 0, tid);
        else
            prep_t1t2(AF, V, out + IM::T1, sm + SM::T2, tid);
        load_taps(item + gridDim.x, (k + 1) & 1);      // the next item's taps, in flight from here
        if (tid < 64) reinterpret_cast<float*>(out + IM::VEC)[tid] = V.dcy[tid] * V.ik[tid];
        else if (tid == 64) reinterpret_cast<float*>(out + IM::VEC)[64] = V.gam[L - 1];
        fence_async_smem();
        tc_fence_before();
        named_sync(1, PREP_THREADS);
        if (tid == 0) {   // P2b: K^T T2^T -> XW
            tc_fence_after();
            const uint64_t dKmn = sw128_desc(smem_u32(KQ), 16384, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tb + TM_XW, dKmn + (uint64_t)(kk * 2048 >> 4), dT2 + (uint64_t)(kk * 32 >> 4), ID_MNK,
                            kk > 0);
            mma_commit(&bars[3]);
            ++n2;
        }
        prep_qtilde<DK>(KQ, V, tid);                    // P1 has read Q; P2b reads only K
        fence_async_smem();
        named_sync(1, PREP_THREADS);
        if (tid == 0) {
#pragma unroll
            for (int kb = 0; kb < NKB; ++kb) bulk_store(out + IM::Q + kb * 8192, KQ + kb * 16384 + 8192, 8192);
            bulk_commit();
        }
        if (!(ok = __syncthreads_and(mbar_wait(&bars[3], (uint32_t)k & 1)))) break;
        // P2b has read K: once the Q~ copy has read Q, the tile is free for a later item
        if (tid == 0 && item + PREP_KQBUF * (int)gridDim.x < n_items) {
            bulk_wait_read_all();
            issue_load(item + PREP_KQBUF * gridDim.x, buf);
            ++nld[buf];
        }
        tc_fence_after();
        prep_wt<DK>(tb + TM_XW, out + IM::WT, tid);
        tc_fence_before();
        named_sync(1, PREP_THREADS);                    // XP, XW and T2 free for the next item
    }
    if (tid == 0) {
        bulk_wait_all();             // shared memory stays valid until the copies have read it
        if (!ok) {                   // a wait ran out: let issued loads / MMAs finish (bounded)
            for (int q = 0; q < PREP_KQBUF; ++q)
                if (nld[q] > ndone[q]) mbar_wait(&bars[q], (uint32_t)(nld[q] - 1) & 1);
            if (n1 > 0) mbar_wait(&bars[2], (uint32_t)(n1 - 1) & 1);
            if (n2 > 0) mbar_wait(&bars[3], (uint32_t)(n2 - 1) & 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid < 32) tmem_dealloc(tb, 128);
}

}  // namespace pfws
}  // namespace jet
