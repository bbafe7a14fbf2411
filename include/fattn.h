/*
 * fattn.h -- C ABI of libfattn: exact, IO-aware scaled-dot-product attention on B200 (sm_100a).
 *
 * The operation (systems-analysis.info "FlashAttention (PL)", section "Problematyka standardowego
 * mechanizmu uwagi"; chipfoundryservices.com glossary "Flash Attention", first paragraph):
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V,      L_i = ln sum_j exp(scale * q_i . k_j)
 *
 * computed tile by tile with the online-softmax recurrence (chipfoundryservices.com glossary,
 * "Tiling Algorithm" steps 1-6; robocikowo.com "Flash Attention", the running max m and sum l and
 * the update O <- rescale(O_prev, m_old, m_new) + exp(S_new - m_new) V_j), so the N x N score
 * matrix is never written to device memory.  The backward recomputes P from the saved L instead
 * of storing it (robocikowo.com "Flash Attention": backward by recomputation from O and L).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are DEVICE pointers, contiguous, row-major:
 *      q, k, v, o, dO, dq, dk, dv : bfloat16 [B, H, N, d]   (element (b,h,n,c) at ((b*H+h)*N+n)*d+c)
 *      lse                        : float32  [B, H, N]      natural-log logsumexp of the scaled
 *                                                            scores of each query row
 *  - Every pointer must be 16-byte aligned (the kernels read and write through the Tensor Memory
 *    Accelerator); a misaligned pointer returns FA_ERR_MISALIGNED before any launch.
 *  - d must be 64, 128 or 256; any N >= 1 is accepted (rows past N are masked, stores clipped).
 *  - causal != 0 hides key j from query i when j > i (N_q = N_k, so both alignments agree).
 *  - scale is the factor applied to q.k (1/sqrt(d) in the usual use); it must be finite and > 0.
 *  - The caller owns and allocates every buffer, including the backward workspace; the library
 *    allocates no device memory on these paths.  It keeps only host-side caches (device
 *    attributes, resolved driver entry points).
 *  - stream is a cudaStream_t (NULL = legacy default stream).  All work is enqueued
 *    asynchronously on it; no call synchronises the host.
 *  - Return value: FA_OK (0) or an fa_status code.  Argument errors are detected on the host
 *    before anything is launched; a failed launch returns FA_ERR_CUDA.  fa_last_error() gives a
 *    message for the last non-OK status returned on the calling thread.
 *  - Every wait inside the kernels is bounded in time.  If one ever expires (it does not in
 *    correct operation), the kernel records FA_ERR_TIMEOUT in a device status word and returns
 *    instead of hanging; fa_device_status() reads and clears that word.
 */
#ifndef FATTN_H_
#define FATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, B/H/N < 1, non-finite or non-positive scale, size overflow */
  FA_ERR_UNSUPPORTED = 2, /* d not in {64, 128, 256}, or no sm_100 device current */
  FA_ERR_MISALIGNED = 3,  /* a tensor pointer is not 16-byte aligned */
  FA_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed (message in fa_last_error) */
  FA_ERR_TIMEOUT = 5,     /* a kernel gave up on a bounded wait (reported by fa_device_status) */
  FA_ERR_WORKSPACE = 6    /* workspace pointer null/misaligned or smaller than fa_bwd_workspace_size */
} fa_status;

/*
 * fa_fwd -- forward pass.  Writes o = softmax(scale*q k^T [masked]) v (bf16, rounded once from
 * the fp32 accumulator after the final division by the row sum, "Tiling Algorithm" step 6) and
 * lse = m + ln l per query row (fp32; robocikowo.com: L is kept for the backward).
 * Inputs q, k, v are read only.  o and lse are fully overwritten.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd needs for this shape:
 * an fp32 dQ accumulator [B,H,N,d] plus two fp32 row vectors [B,H,roundup(N,128)]
 * (the logsumexp in base 2 and D_i = sum_c dO_ic O_ic), and for d = 64 and 128 a further 32
 * bytes per padded row (the same statistics laid out as a tensor-core operand).  Returns 0 for invalid
 * sizes.
 * The workspace is O(N) per head: no N x N buffer exists on any path.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd -- backward pass.  Given the forward's inputs, its outputs o and lse, and the upstream
 * gradient dO, writes dq, dk, dv (bf16, overwritten, never accumulated into).  P is recomputed
 * from lse (robocikowo.com "Flash Attention": backward by recomputation); then
 *   dV = P^T dO, dP = dO V^T, D = rowsum(dO * o), dS = P * (dP - D), dQ = scale dS K,
 *   dK = scale dS^T Q.
 * o and lse must come from fa_fwd on the same q, k, v, causal and scale.
 * workspace: device pointer, 16-byte aligned, at least fa_bwd_workspace_size(B,H,N,d) bytes,
 * owned by the caller; its contents on entry are ignored and on exit are unspecified.
 * Calls that share a workspace must not overlap on the GPU.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv,
           int B, int H, int N, int d, int causal, float scale,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd_noalloc -- the backward pass for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it is an interface addition of this library.
 *
 * Who needs it: a program whose own pooled allocator already holds nearly all of the GPU's
 * memory (a direct cudaMalloc would fail or fragment that pool), or a host application that
 * forbids allocation while it runs a step, for latency or memory-accounting reasons, cannot
 * provide the workspace fa_bwd asks for.  This variant takes the same tensors as fa_bwd, minus
 * the workspace, and uses a scratch array compiled into the library instead.
 *
 * The scratch is a file-scope static device array of FA_NOALLOC_SCRATCH_BYTES (32 MiB).  Every
 * GPU on which the library's kernels are loaded holds that array until the process exits.
 * Shapes whose fa_bwd_workspace_size exceeds it return FA_ERR_WORKSPACE before any launch
 * (for example B=8, H=12, N=1024, d=64 needs about 29 MB and fits; B=2, H=16, N=8192, d=128
 * needs 145 MB and does not).  The entry point calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream capture.
 * The cached address belongs to the device's primary context, which the CUDA runtime keeps for
 * the life of the process: a caller that resets the device (cudaDeviceReset) or drives the
 * library from another context on the same device invalidates it, and must not call this
 * entry point afterwards.
 * All calls on a device share the one array, which keeps whatever the last call left in it
 * (the kernels clear what must start at zero).  Calls that overlap on the GPU -- on different
 * streams, or from different host threads -- race on the array and corrupt each other's
 * results: serialise them.  Arguments, layouts and results are otherwise those of fa_bwd.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * fa_fwd_fp8 -- forward pass on FP8 inputs, the low-precision forward the pages attribute to
 * FlashAttention-3 (robocikowo.com "Flash Attention", the FA-3 entry; systems-analysis.info
 * "FlashAttention (PL)", section "FlashAttention-3 (2024)"; dexblog.ro, the dtype row: FP8 in
 * the forward).  The attended tensors are q_scale*Q8, k_scale*K8 and v_scale*V8:
 *     O = softmax(scale * (q_scale Q8)(k_scale K8)^T [masked]) (v_scale V8),  L as for fa_fwd.
 *   q8, k8, v8 : e4m3 codes [B, H, N, d], one byte per element (1 sign, 4 exponent bits with
 *                bias 7, 3 mantissa bits; S.1111.111 is NaN and must not occur)
 *   q_scale, k_scale, v_scale : per-tensor factors, finite and > 0 (else FA_ERR_INVALID_ARG)
 *   o          : bfloat16 [B, H, N, d];  lse : float32 [B, H, N] (natural log, as for fa_fwd)
 * Both GEMMs run on e4m3 operands with fp32 accumulation; the softmax weights are rounded to
 * e4m3 (scaled so the largest weight of a row is 256, exactly representable) before they
 * multiply V8, so O carries that rounding -- at most 2^-4 of sum_j P_ij |v_j| per element,
 * usually far less -- while lse is computed from the fp32 exponentials.  Layout, alignment,
 * ownership, streams and errors as for fa_fwd (no backward: the pages name FP8 for the forward).
 */
int fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale, float k_scale,
               float v_scale, void* o, float* lse, int B, int H, int N, int d, int causal,
               float scale, void* stream);

/*
 * Grouped-query attention (GQA): H query heads share H_kv key/value heads.  H_kv = 1 is the
 * multi-query attention (MQA) that systems-analysis.info "FlashAttention (PL)", section
 * "FlashAttention-2 (2023)", lists among the second version's additions; H_kv between 1 and H
 * generalises it.  Query head h reads key/value head h / (H / H_kv): consecutive groups
 * of H / H_kv query heads share one.  The result is exactly that of fa_fwd / fa_bwd on K and V
 * with each key/value head repeated H / H_kv times, without materialising the copies.
 *   q, o, dO, dq : bfloat16 [B, H, N, d]        lse : float32 [B, H, N]
 *   k, v, dk, dv : bfloat16 [B, H_kv, N, d]
 * dk and dv hold the gradient summed over the H / H_kv query heads that read each key/value
 * head.  H_kv must divide H (else FA_ERR_INVALID_ARG).  The backward's workspace is
 * fa_bwd_gqa_workspace_size(B, H, H_kv, N, d) bytes: fa_bwd_workspace_size's, plus, when H_kv < H,
 * two fp32 [B, H_kv, N, d] accumulators.  They are used when there are too few (key block,
 * key/value head) pairs to fill the GPU: a group's query heads are then dealt out to several
 * CTAs whose dK, dV sums meet in fp32 (so dk and dv are not bitwise reproducible run to run in
 * that case).  Every other convention -- alignment, ownership, streams, errors -- is that of
 * fa_fwd / fa_bwd, which are these calls with H_kv = H.
 */
size_t fa_bwd_gqa_workspace_size(int B, int H, int H_kv, int N, int d);
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int H, int H_kv, int N, int d, int causal, float scale, void* stream);
int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv,
               int B, int H, int H_kv, int N, int d, int causal, float scale,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Split-key forward with a logsumexp merge (decoding and other shapes with few query blocks, or
 * queries and keys of different lengths).  The keys of each head are cut into `splits` ranges
 * of whole 128-key tiles that run as separate work units; each writes a partial output and
 * logsumexp, and a merge kernel combines them exactly by the associativity of the online-softmax
 * update (robocikowo.com "Flash Attention": O <- rescale(O_prev, m_old, m_new) + ...;
 * chipfoundryservices.com glossary "Online Softmax Trick"):  L = ln sum_s exp(L_s),
 * O = sum_s exp(L_s - L) O_s.  The result is that of the plain definition.
 *   q, o : bfloat16 [B, H, Nq, d]     lse : float32 [B, H, Nq]
 *   k, v : bfloat16 [B, H_kv, Nk, d]  (H_kv divides H, as for fa_fwd_gqa)
 * causal != 0 aligns the queries with the END of the keys: query i sees keys j <= i + Nk - Nq
 * (the last query sees every key, as a decoding step does); it needs Nq <= Nk.
 * splits >= 1 is the requested number of ranges; it is reduced to the number of key tiles,
 * ceil(Nk / 128), and to the ranges that stay non-empty.  With one range nothing is merged and
 * no workspace is needed.  Otherwise workspace is a caller-owned device buffer, 16-byte
 * aligned, of at least fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, splits) bytes (fp32
 * partial outputs and logsumexps); its contents on entry are ignored.  Calls that share a
 * workspace must not overlap on the GPU.  Errors as for fa_fwd, plus FA_ERR_INVALID_ARG for
 * splits < 1 or causal with Nq > Nk, and FA_ERR_WORKSPACE for a missing or short workspace.
 */
size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int splits);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int H_kv, int Nq, int Nk, int d, int causal, float scale,
                   int splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Partial results and their merge: the building blocks of ring (context-parallel) attention,
 * where each rank holds a shard of the sequence and the key/value shards travel around the
 * ranks.  A query shard's attention over all keys is assembled from its attention over each key
 * shard by the associativity of the online-softmax update (robocikowo.com "Flash Attention": the
 * rescale rule; chipfoundryservices.com glossary "Impact on Sequence Length": the method is what
 * lets the sequence grow; the ring across GPUs is this library's extension of it).
 *
 * fa_fwd_partial -- attention of Nq queries against Nk keys (as for fa_fwd_splitkv: q [B, H, Nq,
 * d] bf16, k and v [B, H_kv, Nk, d] bf16, causal aligned to the END of the keys and needing
 * Nq <= Nk), written unrounded: o_part fp32 [B, H, Nq, d] (normalised over these keys only) and
 * lse_part fp32 [B, H, Nq] (natural log; -inf for a row that sees none of the keys, whose o_part
 * row is then 0).  Errors as for fa_fwd_splitkv.
 *
 * fa_merge_partials -- o bf16 [rows, d] and lse fp32 [rows] from n_parts partial results
 * o_parts fp32 [n_parts, rows, d] and lse_parts fp32 [n_parts, rows] of the same query rows
 * over disjoint key sets: lse = ln sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s, exactly
 * the attention over the union of the key sets.  rows is B*H*Nq of the partials.  d must be 64,
 * 128 or 256; n_parts, rows >= 1; 16-byte aligned pointers.
 */
int fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                   int B, int H, int H_kv, int Nq, int Nk, int d, int causal, float scale,
                   void* stream);
int fa_merge_partials(const float* o_parts, const float* lse_parts, int n_parts, void* o,
                      float* lse, long long rows, int d, void* stream);

/*
 * fa_fwd_bwd_host -- forward and backward from HOST buffers, for callers whose tensors live in
 * host memory.  The B*H heads are independent, so they are cut into `chunks` groups of
 * consecutive heads: while group c runs fa_fwd + fa_bwd on `stream`, group c+1's inputs are
 * copied to the device and group c-1's results back, on two copy streams of the library's own
 * (host-side objects created once per device), so the PCIe transfers overlap the kernels.
 *   q, k, v, dO      : host bfloat16 [B, H, N, d] inputs (pinned, e.g. cudaHostAlloc'd, for the
 *                      copies to run asynchronously; pageable memory works but serialises them)
 *   dq, dk, dv       : host bfloat16 [B, H, N, d] outputs; o (bf16) and lse (fp32 [B, H, N]) are
 *                      optional outputs (NULL: not copied back)
 *   device_buffer    : caller-owned device memory, 256-byte aligned, of at least
 *                      fa_fwd_bwd_host_device_bytes(B, H, N, d, chunks) bytes (device copies of
 *                      every tensor plus one group's backward workspace); contents unspecified
 *   chunks           : 1 .. B*H (1: no overlap)
 * The work starts after what is already queued on `stream` and the host outputs are complete
 * when `stream` is; synchronise `stream` before reading them.  One head per key/value head only
 * (no grouped heads).  Calls on one device must not overlap (they share the copy streams and
 * events).  Errors as for fa_fwd / fa_bwd, FA_ERR_INVALID_ARG for chunks outside 1..B*H, and
 * FA_ERR_WORKSPACE for a missing, misaligned or short device buffer.
 */
size_t fa_fwd_bwd_host_device_bytes(int B, int H, int N, int d, int chunks);
int fa_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dO,
                    void* o, float* lse, void* dq, void* dk, void* dv,
                    int B, int H, int N, int d, int causal, float scale, int chunks,
                    void* device_buffer, size_t device_bytes, void* stream);

/* Message for the last non-OK status returned on this host thread ("" if none). */
const char* fa_last_error(void);

/*
 * fa_device_status -- synchronises `stream`, then reads and clears the device status word of
 * the current device.  Returns FA_OK, FA_ERR_TIMEOUT if a kernel abandoned a bounded wait since
 * the last call, FA_ERR_UNSUPPORTED if a kernel found its shared memory placed so that its tiles
 * could not be aligned and did no work, or FA_ERR_CUDA if the synchronisation itself failed.
 */
int fa_device_status(void* stream);

/*
 * fa_selftest_exp2_fma -- test support, not part of the attention computation: y[i] = 2^x[i] for
 * n floats (device pointers) as computed by the FP8 forward's FMA-pipe exponential (argument
 * reduction n = round(x), f = x - n, our own cubic for 2^f with relative error at most 7.5e-5 on
 * [-1/2, 1/2]; inputs below -126 are clamped there).  Lets a test check the device function
 * against exp2 with that bound.  Errors: FA_ERR_INVALID_ARG for null pointers or n < 0.
 */
int fa_selftest_exp2_fma(const float* x, float* y, int n, void* stream);

/* Library version as major*10000 + minor*100 + patch. */
int fa_version(void);

/*
 * Benchmark support: per-kernel device time.  Not part of the attention computation.
 * fa_timer_enable(on != 0) makes every later kernel launch of the library record a pair of CUDA
 * events around itself on its launching stream (host-side objects only; no device memory).
 * fa_timer_read(kernel, &launches, &total_ms) waits for the recorded events of one kernel kind,
 * returns the number of launches and their summed device time, and forgets them.
 * Kernel kinds: FA_KERNEL_FWD, FA_KERNEL_BWD_PRE, FA_KERNEL_BWD_MAIN, FA_KERNEL_BWD_POST,
 * FA_KERNEL_FWD_MERGE (the split-key merge of fa_fwd_splitkv).
 */
enum { FA_KERNEL_FWD = 0, FA_KERNEL_BWD_PRE = 1, FA_KERNEL_BWD_MAIN = 2, FA_KERNEL_BWD_POST = 3,
       FA_KERNEL_FWD_MERGE = 4 };
int fa_timer_enable(int on);
int fa_timer_read(int kernel, int* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* FATTN_H_ */
