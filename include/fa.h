/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * What it computes.  Exact scaled-dot-product attention,
 *     O = softmax(scale * Q K^T  [+ causal mask]) V,
 * with the per-row logsumexp, and its gradients.  The computation is tiled
 * through on-chip memory and never writes the N x N score matrix to HBM
 * ("FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness", sections "Ideas clave: Tiling" and "Softmax en linea";
 * "FlashAttention" (aiunderstanding.org), section "Apercu technique").  The
 * backward pass recomputes the attention blocks from Q, K and the stored
 * logsumexp instead of storing them (same AI Atlas page, "Recalcular en vez de
 * guardar"; "FlashAttention" (freenetmedia.pl), section "Jak dzialaja
 * FlashAttention?").  Packed variable-length batches follow "Flash Attention"
 * (docs.monostate.ai), section "Con Sequence Packing": each packed sequence
 * attends only to itself.
 *
 * Conventions (the pages give no equations; these are the plain readings):
 *   - scale is a caller-supplied float, normally 1/sqrt(d);
 *   - causal: query i sees key j iff j <= i, positions local to the sequence;
 *   - LSE_i = ln sum_j exp(scale * q_i . k_j) over unmasked j (natural log);
 *   - dense tensors Q, K, V, O, dO, dQ, dK, dV: contiguous bf16 [B, N, H, d]
 *     (head dim innermost); dense LSE and the D vector: fp32 [B, H, N];
 *   - packed tensors: contiguous bf16 [total, H, d]; packed LSE: fp32 [H, total];
 *     cu_seqlens: int32 device array of nseq+1 non-decreasing prefix offsets
 *     with cu_seqlens[0] = 0 and cu_seqlens[nseq] = total;
 *   - head dim d is 64 or 128; bf16 inputs, fp32 accumulation and softmax.
 *
 * Ownership.  Every pointer is a DEVICE pointer owned by the caller, 16-byte
 * aligned, on the current CUDA device.  No call allocates device memory:
 * the backward pass takes a caller-allocated workspace of
 * fa_bwd_workspace_size() bytes (fa_bwd_noalloc instead uses a fixed static
 * array in the library's device image).  Outputs are fully overwritten; the
 * workspace holds no state between calls.  All calls are asynchronous on
 * `stream` (a cudaStream_t; NULL = legacy default stream) and return after
 * the launch; errors found on the host are returned before anything is
 * launched.  Calls are thread-safe.
 *
 * Errors.  FA_ERR_INVALID_ARG for a null or misaligned pointer or a size < 1
 * or too large; FA_ERR_WORKSPACE for a workspace smaller than the call needs
 * (and, in fa_bwd_noalloc, a problem larger than its static scratch);
 * FA_ERR_UNSUPPORTED for d not in
 * {64, 128} or a device that is not compute capability 10.0 (sm_100); FA_ERR_CUDA
 * when a CUDA call or launch fails.  Every on-device pipeline wait is bounded:
 * an expired wait ends the kernel and sets a device error word, which
 * fa_get_device_error() reports as FA_ERR_TIMEOUT.  The library never calls
 * exit, abort or __trap.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,
  FA_ERR_UNSUPPORTED = 2,
  FA_ERR_CUDA = 3,
  FA_ERR_TIMEOUT = 4,
  FA_ERR_WORKSPACE = 5
} fa_status;

/* Forward, dense batch.
 * q, k, v: bf16 [B, N, H, d] inputs.  o: bf16 [B, N, H, d] output.
 * lse: fp32 [B, H, N] output (natural-log logsumexp of each query row).
 * causal: 0 or 1.  One fused kernel; no N x N buffer exists at any point. */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int N, int H, int d, float scale, int causal, void* stream);

/* Forward, packed variable-length batch.
 * q, k, v, o: bf16 [total, H, d]; lse: fp32 [H, total]; cu_seqlens: int32
 * device array [nseq + 1]; max_seqlen >= every sequence length (used to size
 * the launch; sequences longer than it are an error the kernel cannot see,
 * so pass the true maximum). */
fa_status fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens, int nseq, int total, int max_seqlen,
                        int H, int d, float scale, int causal, void* stream);

/* Bytes of workspace the backward pass needs for rows = B*N (dense) or
 * rows = total (packed): an fp32 dQ accumulator [rows, H, d] plus the fp32
 * D = rowsum(dO * O) vector [rows * H], each 256-byte aligned.  Returns 0
 * for invalid sizes. */
size_t fa_bwd_workspace_size(int B, int N, int H, int d);

/* Backward, dense batch.
 * q, k, v, o, dO: bf16 [B, N, H, d] (o and lse exactly as fa_fwd returned them);
 * lse: fp32 [B, H, N].  dq, dk, dv: bf16 [B, N, H, d] outputs.
 * workspace: device buffer of ws_bytes >= fa_bwd_workspace_size(B, N, H, d).
 * P is recomputed tile by tile from Q, K and lse; dQ is accumulated in fp32
 * in the workspace and cast to bf16 at the end. */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                 int B, int N, int H, int d, float scale, int causal, void* stream);

/* Backward, packed variable-length batch.  Layouts as fa_varlen_fwd;
 * ws_bytes >= fa_bwd_workspace_size(1, total, H, d). */
fa_status fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                        const int* cu_seqlens, int nseq, int total, int max_seqlen,
                        int H, int d, float scale, int causal, void* stream);

/* Deterministic backward, dense batch ("FlashAttention-2 (PT)", section
 * "Desempenho e eficiencia": the method is exact and deterministic).
 * Arguments, layouts, workspace size and errors are those of fa_bwd.  The
 * outputs are bitwise reproducible from run to run: dK and dV come from the
 * same fused pass (without its dQ product), and dQ from a second pass in
 * which one CTA per 128-row query tile sums the key tiles in increasing
 * order in tensor memory (S and dP are recomputed there; no atomics).  Only
 * the D part of the workspace is used.  About 1.4x the matrix work of
 * fa_bwd. */
fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                               int B, int N, int H, int d, float scale, int causal, void* stream);

/* Deterministic backward, packed variable-length batch.  Arguments as
 * fa_varlen_bwd; results bitwise reproducible as for fa_bwd_deterministic. */
fa_status fa_varlen_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                      const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                      void* workspace, size_t ws_bytes, const int* cu_seqlens, int nseq,
                                      int total, int max_seqlen, int H, int d, float scale, int causal,
                                      void* stream);

/* Bytes of workspace fa_fwd_fp8 needs: V transposed to e4m3 [B, H, 128,
 * Npad] with Npad = N rounded up to a multiple of 16, 256-byte aligned.
 * 0 for invalid sizes (d must be 128). */
size_t fa_fwd_fp8_workspace_size(int B, int N, int H, int d);

/* Forward with 8-bit inputs ("FlashAttention-2 (PT)", section
 * "FlashAttention-3": FP8 support).  q, k, v: e4m3 (OCP FP8, bias 7, no
 * infinities) [B, N, H, 128]; the inputs the attention is taken of are
 * descale_q * q, descale_k * k and descale_v * v (each descale finite and
 * > 0).  o: bf16 [B, N, H, 128]; lse: fp32 [B, H, N] (natural log) of those
 * scaled inputs.  Scores are exact products accumulated in fp32; P is
 * rounded to e4m3 for the P V product (relative error <= 2^-4 per entry
 * above 2^-6, absolute <= 2^-10 below) while the row sums use the unrounded
 * P.  workspace: device buffer of ws_bytes >= fa_fwd_fp8_workspace_size(),
 * 256-byte aligned (holds V^T for the call).  Dense batches only; d must be
 * 128 (FA_ERR_UNSUPPORTED otherwise); B and H at most 65535
 * (FA_ERR_INVALID_ARG otherwise). */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k,
                     float descale_v, void* o, float* lse, void* workspace, size_t ws_bytes,
                     int B, int N, int H, int d, float scale, int causal, void* stream);

/* Bytes of workspace fa_decode_fwd needs (per-entry tile offsets and fp32
 * partial outputs and logsumexps of cache segments shared by two or more
 * CTAs; 256-byte aligned; it depends on B, Nq and d only).  0 for invalid
 * sizes. */
size_t fa_decode_workspace_size(int B, int Nq, int Nk, int H, int d);

/* Decode-shaped forward: Nq new queries per batch entry (1 <= Nq <= 16)
 * against a cache of up to Nk keys and values.  The method's tiling and
 * online softmax ("FlashAttention: Fast and Memory-Efficient Exact
 * Attention with IO-Awareness", sections "Tiling" and "Softmax en linea")
 * applied over equal shares of all the cache tiles in parallel (one share
 * per CTA, whatever the per-sequence lengths), the pieces of a sequence that
 * falls on several shares merged exactly through their logsumexps.
 * q, o: bf16 [B, Nq, H, d]; k_cache, v_cache: bf16 [B, Nk, H, d];
 * lse: fp32 [B, H, Nq] output (natural log).
 * seqlens_k: int32 device array [B] of valid cache rows per batch entry
 * (0 <= L_b <= Nk), or NULL for all Nk; rows past L_b are never used in the
 * arithmetic (they may hold anything).  If any value is outside [0, Nk]
 * the call writes no output and fa_get_device_error() reports
 * FA_ERR_INVALID_ARG.
 * causal = 1: query i is the token at position L_b - Nq + i and sees keys
 * j <= L_b - Nq + i; a query that sees no key gets O = 0 and LSE = -inf.
 * workspace: device buffer of ws_bytes >= fa_decode_workspace_size(...),
 * 256-byte aligned.
 * Returns FA_ERR_UNSUPPORTED for Nq > 16 or d not in {64, 128}, and
 * FA_ERR_INVALID_ARG for B or H above 65535 (the launch grid's limits). */
fa_status fa_decode_fwd(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                        const int* seqlens_k, void* workspace, size_t ws_bytes,
                        int B, int Nq, int Nk, int H, int d, float scale, int causal, void* stream);

/* Measurement hook (no counterpart in the method: it serves the roofline
 * measurement, which times the dominant kernel of a multi-kernel call on its
 * own).  events: n (1..8) cudaEvent_t handles, created by the caller on the
 * current device and owned by it.  The NEXT compute call made by this host
 * thread records events[0] on that call's stream just before its first kernel
 * launch and events[i] right after its i-th launch, as far as n reaches; the
 * hook is then cleared, whether that call succeeded or not.  For fa_bwd the
 * launches are: D / accumulator preprocess, the fused main kernel, the dQ
 * conversion.  FA_ERR_INVALID_ARG for a null array or entry, or n outside
 * 1..8.  Recording an event adds no work to the kernels themselves. */
fa_status fa_record_launch_events(void* const* events, int n);

/* Backward pass, dense batch, for callers that cannot allocate device memory.
 * There is no counterpart to this in the method's description: it exists for
 * callers that may not call cudaMalloc (or any allocating routine) when they
 * run the backward pass -- for example code running inside an allocator or
 * memory-pool callback, or a runtime with a fixed, pre-planned memory budget.
 * Arguments and results are those of fa_bwd without the workspace: the fp32
 * scratch comes from one static device array of FA_STATIC_SCRATCH_BYTES that
 * the library image carries on every GPU that loads it (held until exit).
 * Nothing is allocated or freed by this call.
 *   - Problems needing more than FA_STATIC_SCRATCH_BYTES of scratch
 *     (fa_bwd_workspace_size(B, N, H, d) > FA_STATIC_SCRATCH_BYTES) are
 *     rejected with FA_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     the parts that must start at zero are cleared by each call itself.
 *     Calls whose GPU work overlaps (different streams, or different host
 *     threads without ordering) race on the array: serialise them. */
#define FA_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv,
                         int B, int N, int H, int d, float scale, int causal, void* stream);

/* Static text for a status code (never NULL). */
const char* fa_status_string(fa_status s);

/* Synchronises `stream`, then reads and clears this device's error word.
 * FA_ERR_TIMEOUT if a kernel gave up on a bounded wait since the last call;
 * otherwise FA_ERR_INVALID_ARG if a kernel found device-side sizes that
 * contradict the call (cu_seqlens offsets past `total` or longer than
 * max_seqlen, seqlens_k outside [0, Nk]) and skipped that work;
 * FA_ERR_CUDA if the synchronisation itself failed; else FA_OK. */
fa_status fa_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
