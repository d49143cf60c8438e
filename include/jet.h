/*
 * jet.h — C ABI of the JetBlock token mixer on NVIDIA B200 (sm_100a).
 *
 * The mixer (Jet-Nemotron, "JetBlock"):
 *   1. kernel generator   w_t = SiLU(x_t W1) W2          d_model -> 32 -> H*4
 *   2. dynamic causal conv on V, width 4:
 *        v'_t[h,:] = sum_{j=0..3} w_t[h,j] v_{t-j}[h,:]   (tap 0 = current token)
 *   3. Gated DeltaNet on L2-normalised q, k (no 1/sqrt(dk) scale):
 *        S_t = a_t (S_{t-1} - b_t (S_{t-1} k_t) k_t^T) + b_t v'_t k_t^T,
 *        o_t = S_t q_t,   a_t = exp(g_t) (g_t <= 0),  b_t in (0,1),  S in R^{dv x dk}
 * Sources: Jet-Nemotron paper (arXiv 2508.15884, Chinese translation on
 * adg.csdn.net), section 2.3 "linear attention block selection" (Gated
 * DeltaNet: data-dependent gate + delta rule) and section 2.4 "new attention
 * block design" (kernel generator: linear reduction, SiLU, linear output of
 * the conv taps; dynamic conv applied to V only; no static conv on Q/K); the
 * xugj520.cn explainer, section 2.2 "JetBlock" (q/k dim 96 or 128, v dim 256,
 * 12 or 16 heads, conv kernel 4, generator hidden 32).
 *
 * Conventions for every entry point
 *   - Pointers are caller-owned DEVICE memory (except where stated). The
 *     library never allocates or frees device memory and keeps no state
 *     between calls except a per-device error word (see jet_device_error).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously. Argument checks are synchronous and
 *     happen before any launch: on error nothing is enqueued.
 *   - Layouts are dense row-major, token-major:
 *       x [B,T,D];  q, k [B,T,H,dk];  v, v', o [B,T,H,dv];  g, beta [B,T,H];
 *       W1 [D,hidden];  W2 [hidden,H*width] (column h*width+j = tap j of head h);
 *       conv taps [B,T,H,width] float32;  state S [B,H,dv,dk] float32 (dk fastest);
 *       conv history [B,width-1,H,dv] = raw V of positions -3,-2,-1 (oldest first).
 *   - dtype JET_BF16: x, q, k, v, v', o, W1, W2 and the history are bf16; g, beta,
 *     taps and states are float32; all arithmetic accumulates in float32.
 *     dtype JET_F32: everything float32.
 *   - Alignment: the bulk tensors (x, q, k, v, v', o, histories, states,
 *     workspace) must be 16-byte aligned; g, beta and conv taps 4-byte aligned;
 *     W1 and W2 aligned to their element size. jet_gdn_decode_step needs 16
 *     bytes only for S (its per-token q, k, v, o need element alignment).
 *     Sizes must be > 0 (T may be any length; no multiple of the chunk is
 *     needed) and the element counts must fit in int64.
 *   - Supported shapes: width == 4, hidden == 32, chunk == 64, dk % 16 == 0
 *     and dk <= 128, dv % 32 == 0 and dv <= 256, D % 16 == 0, H <= 64.
 *     Anything else returns JET_ERR_UNSUPPORTED.
 *   - Nothing aborts, exits or throws across the ABI. Thread-safe.
 */
#ifndef JET_H
#define JET_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JET_OK = 0,
    JET_ERR_INVALID_ARG = 1,   /* null required pointer, size <= 0 or overflowing, aliasing */
    JET_ERR_UNSUPPORTED = 2,   /* shape outside the supported set above */
    JET_ERR_MISALIGNED = 3,    /* a pointer below its required alignment */
    JET_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    JET_ERR_TIMEOUT = 5,       /* a bounded in-kernel wait ran out (via jet_device_error) */
    JET_ERR_DEVICE = 6,        /* a kernel flagged bad data (via jet_device_error) */
    JET_ERR_WORKSPACE = 7,     /* workspace pointer null or smaller than required */
    JET_ERR_TOO_LARGE = 8,     /* sizes need more scratch than jet_gdn_prefill_noalloc's fixed buffer */
    JET_ERR_LIBRARY = 9        /* a library the call needs (cuBLAS, for jet_jetblock_layer) could not be loaded */
} jet_status;

typedef enum { JET_F32 = 0, JET_BF16 = 1 } jet_dtype;

/*
 * Kernel generator only (step 1; paper section 2.4): conv_w[b,t,h,j] = w_t[h,j].
 *   x [B,T,D], w1 [D,hidden], w2 [hidden,H*width] in `dt`; conv_w [B,T,H,width] float32 out.
 */
jet_status jet_kernel_gen(const void* x, const void* w1, const void* w2, float* conv_w,
                          int B, int T, int D, int H, int hidden, int width,
                          jet_dtype dt, void* stream);

/*
 * Generator fused with the dynamic causal conv on V (steps 1-2; paper section
 * 2.4), one pass over V.
 *   v [B,T,H,dv] raw values in; v_out [B,T,H,dv] conv output (v') out.
 *   hist_in [B,width-1,H,dv] or NULL: raw V of the 3 positions before token 0
 *     (NULL = zeros, i.e. the start of a sequence).
 *   hist_out [B,width-1,H,dv] or NULL: receives the last 3 raw V positions of
 *     [hist_in, v] (the history for the next call). Must not overlap hist_in.
 *   conv_w_out [B,T,H,width] float32 or NULL: the generated taps.
 * For decode call it with T = 1 and both histories.
 */
jet_status jet_dyn_conv_v(const void* x, const void* w1, const void* w2, const void* v,
                          const void* hist_in, void* v_out, void* hist_out, float* conv_w_out,
                          int B, int T, int D, int H, int dv, int hidden, int width,
                          jet_dtype dt, void* stream);

/*
 * Device workspace of jet_gdn_prefill for these sizes, in bytes (either may
 * be 0). With at least jet_gdn_prefill_workspace_size bytes the prefill runs
 * its fastest plan: every chunk's state-independent part is prepared at once
 * into per-chunk tiles (about 47 KB per chunk of 64 tokens and head at
 * dk = 96, so this grows with B * T * H), then the state chain runs. With
 * at least jet_gdn_prefill_workspace_min bytes (the sequence-parallel
 * segment buffers only, at most a few tens of MB and independent of T beyond
 * a few thousand tokens) it runs a plan that prepares each chunk inside the
 * chain kernel; the results agree within the bf16 tolerance, not bit for bit.
 */
size_t jet_gdn_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt);
size_t jet_gdn_prefill_workspace_min(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt);

/*
 * Gated DeltaNet prefill over T tokens per sequence (step 3; paper section
 * 2.3), chunkwise (chunk = 64) in the WY / UT-transform form; q and k are
 * L2-normalised inside (eps 1e-6 under the square root).
 *   q, k [B,T,H,dk]; v [B,T,H,dv] (normally v' from jet_dyn_conv_v); g, beta [B,T,H] float32.
 *   S0 [B,H,dv,dk] float32 or NULL (zeros). o [B,T,H,dv] out.
 *   S_out [B,H,dv,dk] float32 out: the state after token T-1; may alias S0.
 *   workspace / ws_bytes: at least jet_gdn_prefill_workspace_min(...) bytes,
 *   jet_gdn_prefill_workspace_size(...) for the fastest plan (may be NULL
 *   when the minimum is 0). Contents on entry are ignored.
 * A prefill can be continued: pass its S_out as the next call's S0.
 */
jet_status jet_gdn_prefill(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, void* o, float* S_out,
                           void* workspace, size_t ws_bytes,
                           int B, int T, int H, int dk, int dv, int chunk,
                           jet_dtype dt, void* stream);

/*
 * The whole JetBlock mixer over a prompt (steps 1-3; paper sections 2.3 and
 * 2.4): the kernel generator makes every token's taps, the dynamic causal
 * conv is applied to the raw v, and the chunked gated delta rule runs on the
 * result. On the tensor-core path (bf16, dk in {64, 96, 128}, dv a multiple
 * of 128) the conv is folded into each chunk's UT transform (U = T diag(b) V'
 * is linear in the raw V, with a three-token reach into the previous chunk),
 * so v' is never formed; elsewhere a separate conv pass writes v' into the
 * workspace and the SIMT prefill reads it.
 *   x [B,T,D]; w1 [D,hidden], w2 [hidden,H*width] as in jet_kernel_gen.
 *   q, k [B,T,H,dk]; v [B,T,H,dv] raw (before the conv); g, beta [B,T,H] float32.
 *   hist_in [B,3,H,dv] raw V of the 3 positions before token 0, oldest first,
 *     or NULL (zeros: the start of a sequence).
 *   hist_out [B,3,H,dv] or NULL: the last 3 raw V positions of [hist_in, v]
 *     (the history for the decode steps that follow). Must overlap neither
 *     hist_in nor v.
 *   S0, o, S_out as in jet_gdn_prefill (S_out may alias S0); o must not overlap v.
 *   workspace / ws_bytes: at least jet_jetblock_prefill_workspace_size(...)
 *     bytes (the taps, then the chunk images and segment buffers of the
 *     fastest jet_gdn_prefill plan, or a v' buffer off the tensor-core path);
 *     otherwise JET_ERR_WORKSPACE before any launch. Contents on entry are ignored.
 * o and S_out agree with jet_dyn_conv_v followed by jet_gdn_prefill within
 * the bf16 tolerance (the folded path never rounds v' to bf16), not bit for bit.
 * A history containing Inf or NaN can reach the first chunk of the next
 * sequence in the batch (its values meet zero weights there).
 */
size_t jet_jetblock_prefill_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt);
jet_status jet_jetblock_prefill(const void* x, const void* w1, const void* w2,
                                const void* q, const void* k, const void* v,
                                const void* hist_in, void* hist_out,
                                const float* g, const float* beta, const float* S0,
                                void* o, float* S_out, void* workspace, size_t ws_bytes,
                                int B, int T, int D, int H, int dk, int dv,
                                int hidden, int width, int chunk, jet_dtype dt, void* stream);

/*
 * jet_jetblock_prefill over a batch of sequences of different lengths in one
 * call (chunked prefill of several prompts at once: paper section 3.1 and
 * appendix A.3, throughput measurement). The sequences are packed along the
 * token axis: sequence i holds tokens cu_seqlens[i] .. cu_seqlens[i+1]-1.
 *   cu_seqlens: HOST array of nseq + 1 int32 offsets, cu_seqlens[0] = 0,
 *     strictly increasing (every sequence has at least one token); read during
 *     the call only (the launch plan is made from it on the host).
 *   1 <= nseq <= 256 (more returns JET_ERR_UNSUPPORTED).
 *   x [total,D]; q, k [total,H,dk]; v [total,H,dv] raw; g, beta [total,H]
 *     float32; o [total,H,dv] out (total = cu_seqlens[nseq]).
 *   hist_in / hist_out [nseq,3,H,dv] or NULL; S0 / S_out [nseq,H,dv,dk]
 *     float32 (S0 may be NULL; S_out may alias S0), per sequence as in
 *     jet_jetblock_prefill.
 *   workspace: at least jet_jetblock_prefill_varlen_workspace_size(...) bytes.
 * Tensor-core shapes only (bf16, dk in {64, 96, 128}, dv a multiple of 128).
 * Long sequences run in segments of a common length, chosen so that every
 * segment of every sequence runs at once; the results agree with one
 * jet_jetblock_prefill per sequence within the bf16 tolerance.
 */
size_t jet_jetblock_prefill_varlen_workspace_size(const int* cu_seqlens, int nseq, int H, int dk, int dv, int chunk,
                                                  jet_dtype dt);
jet_status jet_jetblock_prefill_varlen(const void* x, const void* w1, const void* w2,
                                       const void* q, const void* k, const void* v,
                                       const void* hist_in, void* hist_out,
                                       const float* g, const float* beta, const float* S0,
                                       void* o, float* S_out, void* workspace, size_t ws_bytes,
                                       const int* cu_seqlens, int nseq, int D, int H, int dk, int dv,
                                       int hidden, int width, int chunk, jet_dtype dt, void* stream);

/*
 * Sequence parallelism over token ranges: one long prompt split into R
 * consecutive ranges, one per GPU. The gated delta rule is affine in the
 * state (paper section 2.3): over a range, S_end = S_start A + E with A the
 * product of the range's per-token transitions and E the end state reached
 * from a zero start, and the range's outputs are affine in S_start too. So
 * every range runs at once from a zero start, the (E, A) pairs are exchanged
 * (all-gather, a few MB per GPU), each range's true start state is composed
 * from them, and a correction adds its term to the outputs. The pages run
 * chunked prefill on one GPU (paper section 3.1 and appendix A.3); the split
 * across GPUs is this library's, built on that affine form.
 *
 * jet_jetblock_prefill_range: the whole mixer over one range (as
 * jet_jetblock_prefill, tensor-core path only: bf16, dk in {64, 96, 128},
 * dv a multiple of 128; else JET_ERR_UNSUPPORTED).
 *   hist_in [B,3,H,dv]: the last three raw V tokens of the previous range (the
 *     conv's halo), or NULL at the start of the sequence.
 *   S0 [B,H,dv,dk] float32 or NULL: the range's start state when known (the
 *     first range), else NULL (zero).
 *   o [B,T,H,dv] out: the outputs for that start state (provisional for
 *     ranges after the first until jet_gdn_range_correct).
 *   E_out [B,H,dv,dk] float32 out: the end state reached from that start.
 *   A_out [B,H,dk,dk] float32 out and Qe_out [B,H,ceil(T/64),64,dk] bf16 out:
 *     the range's transition and output-correction operand; both NULL for
 *     the first range (which needs neither), else both given.
 *   workspace: at least jet_jetblock_prefill_range_workspace_size(...) bytes.
 */
size_t jet_jetblock_prefill_range_workspace_size(int B, int T, int H, int dk, int dv, int chunk, jet_dtype dt);
jet_status jet_jetblock_prefill_range(const void* x, const void* w1, const void* w2,
                                      const void* q, const void* k, const void* v,
                                      const void* hist_in, void* hist_out,
                                      const float* g, const float* beta, const float* S0,
                                      void* o, float* E_out, float* A_out, void* Qe_out,
                                      void* workspace, size_t ws_bytes,
                                      int B, int T, int D, int H, int dk, int dv,
                                      int hidden, int width, int chunk, jet_dtype dt, void* stream);

/*
 * Start states of R ranges from their (E, A) pairs (section 2.3's affine
 * form): S*_1 = E_0, S*_{r+1} = S*_r A_r + E_r, on the tensor cores with
 * float32 accuracy (each operand split into two tf32 parts).
 *   E [R,B,H,dv,dk] float32: E_0 is the first range's true end state, E_r
 *     (r >= 1) the end state of range r from a zero start.
 *   A [R,B,H,dk,dk] float32: the ranges' transitions (entry 0 is not read).
 *   Sb_out [R,B,H,dv,dk] bf16 out: entries 1 .. R-1 receive S*_1 .. S*_{R-1},
 *     the operands of jet_gdn_range_correct (entry 0 is not written).
 *   S_out [B,H,dv,dk] float32 out: the final state S*_R.
 * R >= 2; dk in {64, 96, 128}; dv a multiple of 16, at most 256.
 */
jet_status jet_gdn_range_compose(const float* E, const float* A, void* Sb_out, float* S_out,
                                 int R, int B, int H, int dk, int dv, void* stream);

/*
 * Adds a range's start-state term to its outputs: o += Qe S*^T per chunk of
 * 64 tokens (the outputs are affine in the start state).
 *   Qe [B,H,ceil(T/64),64,dk] bf16: from jet_jetblock_prefill_range.
 *   Sb [B,H,dv,dk] bf16: the range's start state (an entry of Sb_out).
 *   o [B,T,H,dv] bf16, updated in place (must not overlap Qe or Sb).
 * Tensor-core shapes only, as jet_jetblock_prefill_range.
 */
jet_status jet_gdn_range_correct(const void* Qe, const void* Sb, void* o, int B, int T, int H, int dk, int dv,
                                 jet_dtype dt, void* stream);

/*
 * One decode step (step 3 for a single new token per sequence; paper section
 * 2.3, the gated delta rule applied to one token; section 2.5, finding 4:
 * decode cost is set by the state's size), updating S in place:
 *   u = S k,  S' = a S + (b v - a b u) k^T,  o = S' q.
 *   q, k [B,H,dk]; v [B,H,dv] (v' of the new token); g, beta [B,H] float32;
 *   S [B,H,dv,dk] float32 in/out; o [B,H,dv] out.
 */
jet_status jet_gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, float* S, void* o,
                               int B, int H, int dk, int dv, jet_dtype dt, void* stream);

/*
 * jet_gdn_decode_step with the dynamic causal conv of the new token fused in
 * (paper sections 2.3 and 2.4): from the token's generated taps (as made by
 * jet_kernel_gen) and the raw history, v' = w0 v_t + w1 v_{t-1} + w2 v_{t-2}
 * + w3 v_{t-3} (rounded to the storage type), the history is shifted, and S
 * is updated in place, in one pass over S.
 *   q, k [B,H,dk]; v [B,H,dv] raw; hist_in [B,3,H,dv] raw, oldest first, or
 *   NULL (zeros); hist_out [B,3,H,dv] out (must not overlap hist_in);
 *   taps [B,H,4] float32 (16-byte aligned); g, beta [B,H] float32;
 *   S [B,H,dv,dk] float32 in/out; o [B,H,dv] out.
 */
jet_status jet_conv_gdn_decode_step(const void* q, const void* k, const void* v,
                                    const void* hist_in, void* hist_out, const float* taps,
                                    const float* g, const float* beta, float* S, void* o,
                                    int B, int H, int dk, int dv, jet_dtype dt, void* stream);

/*
 * The whole JetBlock mixer for one new token per sequence (steps 1-3 fused;
 * paper sections 2.3 and 2.4): the kernel generator makes the token's taps,
 * the dynamic causal conv is applied to v with the raw history, the history
 * is shifted, and the gated delta rule updates S in place with one read and
 * one write of S. Two launches: the generator + conv (as jet_dyn_conv_v with
 * T = 1, its output v' written into o), then the update (as
 * jet_gdn_decode_step, reading v' from o and writing o over it); the update
 * starts reading its state before the first launch ends.
 *   x [B,D]; w1 [D,hidden], w2 [hidden,H*width] as in jet_kernel_gen;
 *   q, k [B,H,dk]; v [B,H,dv] raw (before the conv); g, beta [B,H] float32;
 *   hist_in [B,3,H,dv] raw history, oldest first, or NULL (zeros);
 *   hist_out [B,3,H,dv] out (must not overlap hist_in);
 *   S [B,H,dv,dk] float32 in/out; o [B,H,dv] out;
 *   taps [B,H,width] float32 out (16-byte aligned): the generated conv taps.
 * v, o and hist_out must not overlap (JET_ERR_INVALID_ARG); v, o and the
 * histories must be 16-byte aligned (JET_ERR_MISALIGNED).
 * Equal bit for bit to jet_dyn_conv_v with T = 1 followed by
 * jet_gdn_decode_step on its output.
 */
jet_status jet_jetblock_decode_step(const void* x, const void* w1, const void* w2,
                                    const void* q, const void* k, const void* v,
                                    const void* hist_in, void* hist_out,
                                    const float* g, const float* beta, float* S, void* o,
                                    float* taps, int B, int D, int H, int dk, int dv,
                                    int hidden, int width, jet_dtype dt, void* stream);

/*
 * jet_jetblock_decode_step over a state cache: the states and conv histories
 * of the running sequences live in caller-owned pools, and entry b of the
 * batch works on pool entry slots[b] in place, so a serving loop never
 * gathers or scatters a state (each is read and written once per step).
 * Two launches: the generator + conv of the new tokens (histories updated in
 * place in hist_pool), then the decode update of S_pool.
 *   x [B,D]; w1, w2 as in jet_kernel_gen; q, k [B,H,dk]; v [B,H,dv] raw;
 *   g, beta [B,H] float32;
 *   hist_pool [n_slots,3,H,dv] (raw histories, oldest first) in/out;
 *   S_pool [n_slots,H,dv,dk] float32 in/out;
 *   slots [B] int32 (device memory) with distinct values in [0, n_slots); a
 *     value outside that range leaves that sequence's outputs and pool
 *     entries untouched and sets the device error word (JET_ERR_DEVICE from
 *     jet_device_error); repeated values race;
 *   o [B,H,dv] out; v_conv [B,H,dv] scratch (the conv output, must not
 *   overlap v); taps [B,H,width] float32 out or NULL.
 * Same arithmetic as jet_dyn_conv_v (T = 1) followed by jet_gdn_decode_step
 * on pool entries gathered into a batch: the results are equal bit for bit.
 */
jet_status jet_jetblock_decode_slots(const void* x, const void* w1, const void* w2,
                                     const void* q, const void* k, const void* v,
                                     const float* g, const float* beta,
                                     void* hist_pool, float* S_pool, const int* slots, int n_slots,
                                     void* o, void* v_conv, float* taps,
                                     int B, int D, int H, int dk, int dv, int hidden, int width,
                                     jet_dtype dt, void* stream);

/*
 * jet_gdn_prefill for callers that cannot allocate device memory. It has no
 * counterpart in the paper; it exists for code that must not call an
 * allocator on its hot path: work recorded into a CUDA graph (allocation is
 * not allowed during stream capture), latency-bound serving loops where an
 * allocation would stall or synchronise the device, and embedders that own a
 * fixed memory budget and hand the library only their input and output
 * buffers.
 *
 * Same operation, arguments and errors as jet_gdn_prefill, minus the
 * workspace: the scratch it needs comes from one fixed array of
 * JET_NOALLOC_SCRATCH_BYTES (16 MiB) inside the library, present on every
 * GPU that loads the library until the process exits. The fastest plan
 * whose scratch fits is used; sizes whose smallest plan needs more
 * (jet_gdn_prefill_workspace_min > JET_NOALLOC_SCRATCH_BYTES) return
 * JET_ERR_TOO_LARGE before anything is launched: the 2B shapes fit at any
 * length (12.5 MB), 16-head dk = 128 shapes longer than 1792 tokens do not
 * (18.0 MB).
 * The first call on a device looks the array's device address up (no
 * allocation) and caches it with the device's current context; the lookup is
 * repeated when that context changes (e.g. after cudaDeviceReset), so make
 * the first call, and the first after such a reset, before any stream
 * capture. The array is
 * shared by all calls on a device and keeps the last call's contents (every
 * element a call reads is written by that call first): calls whose work
 * overlaps on the GPU, e.g. on two streams, race on it and must be ordered
 * by the caller. Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define JET_NOALLOC_SCRATCH_BYTES (16u << 20)
jet_status jet_gdn_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* S0, void* o, float* S_out,
                                   int B, int T, int H, int dk, int dv, int chunk,
                                   jet_dtype dt, void* stream);

/*
 * The JetBlock layer around the mixer (Jet-Nemotron paper, section 2.4: the
 * block takes its queries, keys, values and the generator input from the
 * shared input x; the dynamic conv acts on V alone). The paper gives no form
 * for the gates or the output; this is the Gated DeltaNet layer without its
 * short convolutions:
 *   q = x Wq, k = x Wk, v = x Wv, z = x Wz                 (bf16 GEMMs, float32 accumulate)
 *   g = -softplus(x Wg), beta = sigmoid(x Wb)             (float32)
 *   o = the mixer (jet_jetblock_prefill; for T = 1 the decode kernels, the
 *       state advanced in place in S_out)
 *   y = (o / sqrt(mean_dv(o^2) + 1e-6) * gamma * SiLU(z)) Wo   (per token and head)
 * The six projections and the output projection run on cuBLAS (loaded on the
 * first call; JET_ERR_LIBRARY if it cannot be), the rest in this library.
 *   x [B,T,D] bf16; wq, wk [D,H*dk]; wv, wz [D,H*dv]; wg, wb [D,H];
 *   wo [H*dv,D] (all bf16, row-major); gamma [dv] float32;
 *   w1, w2 the generator's weights as in jet_kernel_gen;
 *   hist_in [B,3,H,dv] or NULL (zeros); hist_out [B,3,H,dv] or NULL (required
 *   for T = 1); S0 [B,H,dv,dk] float32 or NULL (zeros); S_out [B,H,dv,dk]
 *   float32 out (may alias S0); y [B,T,D] bf16 out;
 *   workspace of jet_jetblock_layer_workspace_size bytes (16-byte aligned),
 *   else JET_ERR_WORKSPACE before any launch.
 * bf16 and the tensor-core shapes only (dk in {64, 96, 128}, dv a multiple
 * of 128), D a multiple of 16; else JET_ERR_UNSUPPORTED. cuBLAS is called
 * under a process-wide lock, so concurrent calls from several threads are
 * serialised at their GEMMs.
 */
size_t jet_jetblock_layer_workspace_size(int B, int T, int D, int H, int dk, int dv);
jet_status jet_jetblock_layer(const void* x, const void* wq, const void* wk, const void* wv,
                              const void* wg, const void* wb, const void* wz, const void* wo,
                              const float* gamma, const void* w1, const void* w2,
                              const void* hist_in, void* hist_out, const float* S0, float* S_out,
                              void* y, void* workspace, size_t ws_bytes, int B, int T, int D, int H,
                              int dk, int dv, int hidden, int width, jet_dtype dt, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's error
 * word: JET_ERR_TIMEOUT if a bounded in-kernel wait ran out since the last
 * call, JET_ERR_DEVICE if a kernel flagged bad data, JET_ERR_CUDA if the
 * synchronisation itself failed, else JET_OK.
 */
jet_status jet_device_error(void* stream);

/* Static string naming a status. */
const char* jet_status_string(jet_status s);

/* Number of kernels this library has launched in this process (all devices). */
uint64_t jet_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* JET_H */
