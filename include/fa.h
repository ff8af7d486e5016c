/*
 * Exact tiled softmax attention for NVIDIA B200 (sm_100a): the C ABI.
 *
 * The operation. For every batch b and query head h, with kv = h / (Hq / Hkv):
 *     S = scale * Q[b,h] K[b,kv]^T          (N x N, never written to memory)
 *     S[i,j] = -inf  where causal and j > i
 *     O[b,h] = softmax_rows(S) V[b,kv]
 *     LSE[b,h,i] = log sum_j exp(S[i,j])    (natural log)
 * "FlashAttention: The Algorithm That Made Long-Context AI Possible"
 * (promptingindex.com), section "The quadratic bottleneck in standard
 * attention", defines S = Q K^T and O = softmax(S) V; section "What tiling
 * changes" gives the method: Q, K and V are split into blocks that fit on
 * chip, a running row maximum and a running sum of exponentials make the
 * softmax exact, and the N x N matrix never reaches high-bandwidth memory.
 * "FlashAttention: Fast and Memory-Efficient Exact Attention with
 * IO-Awareness" (abstract) states that the tiled algorithm is exact and needs
 * linear, not quadratic, memory. The scale, the causal mask, the log-sum-exp
 * output and the backward pass are not on those pages; they follow the
 * workload statement the library is built to (scale = 1/sqrt(d) in every
 * shipped workload, causal keeps j <= i).
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers unless said otherwise, 16-byte aligned.
 *   - Tensors are row-major contiguous: Q, O, dO, dQ are [B, Hq, N, d];
 *     K, V, dK, dV are [B, Hkv, N, d]; LSE and D are [B, Hq, N] float32.
 *     bf16 tensors are passed as raw 16-bit storage.
 *   - d is 64, 96 or 128 (96 runs on the 128-column tiles with the extra
 *     columns zero-filled on load and clipped on store; its FLOP cost is
 *     that of 128); the bf16 forwards (fa_fwd, fa_fwd_varlen) also take 192
 *     and 256; each entry point states its own set. N >= 1; Hq is a multiple
 *     of Hkv; scale is finite and > 0.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream), like a
 *     kernel launch; outputs are valid once the stream has been synchronised.
 *   - The caller owns every buffer, workspaces included. The library allocates
 *     no device memory and keeps no state between calls (fa_bwd_noalloc's
 *     built-in scratch array, described at its declaration, is the one
 *     exception).
 *   - Every argument is checked before anything is launched; a failed check
 *     returns an error and launches nothing. A launch error is returned as
 *     FA_ERR_CUDA.
 *   - Not safe to call concurrently on overlapping output buffers.
 */
#ifndef EXACT_TILED_ATTENTION_FA_H
#define EXACT_TILED_ATTENTION_FA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, Hq % Hkv != 0, bad scale */
  FA_ERR_UNSUPPORTED = 2,  /* head dimension not built for this entry point, or a size past the limits */
  FA_ERR_MISALIGNED = 3,   /* a pointer that is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,    /* workspace pointer null or smaller than the *_workspace_size query */
  FA_ERR_CUDA = 5,         /* the CUDA runtime reported an error when launching */
  FA_ERR_TIMEOUT = 6,      /* a kernel gave up on a bounded wait (see fa_last_device_status) */
  FA_ERR_BOUNDS = 7        /* debug library only: a kernel computed a global index outside its buffer */
} fa_status;

/*
 * Forward pass. Writes O (bf16, [B,Hq,N,d]) and LSE (float32, [B,Hq,N],
 * natural log). `lse` may not be null (the backward needs it). d is 64, 96,
 * 128, 192 or 256 (FA_ERR_UNSUPPORTED otherwise); 192 and 256 run one
 * 128-row query tile per CTA over 64-key tiles.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                 cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd needs: D = rowsum(dO * O) and
 * -LSE * log2(e), each float32 [B*Hq, Npad] with Npad = 128 * ceil(N / 128),
 * and the float32 dQ accumulator [B, Hq, N, d], each rounded up to 256
 * bytes. Linear in N. Returns 0 for invalid sizes (fa_bwd's d: 64, 96, 128).
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * Backward pass by recomputation: P is rebuilt from Q, K and the saved LSE,
 * then dV = P^T dO, dP = dO V^T, dS = P * (dP - D), dQ = scale dS K,
 * dK = scale dS^T Q, with dK and dV summed over the Hq / Hkv query heads that
 * share a KV head. `o` and `lse` are fa_fwd's outputs for the same inputs.
 * dq, dk, dv (bf16) are overwritten, not accumulated. The workspace is
 * overwritten; its contents on entry do not matter. d is 64, 96 or 128
 * (FA_ERR_UNSUPPORTED otherwise).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes,
                 int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                 cudaStream_t stream);

/*
 * Packed variable-length batches. The blog page ("FlashAttention: The
 * Algorithm That Made Long-Context AI Possible", section "Version 2 in 2023
 * and version 3 in 2024") notes the method's uptake by training and serving
 * stacks, whose batches pack sequences of different lengths end to end; the
 * pages give no interface. Here every sequence is its own attention problem,
 * exactly as if run alone:
 *   - q, o, dq, dout: [T, Hq, d] bf16 and k, v, dk, dv: [T, Hkv, d] bf16,
 *     token-major, T = total tokens; lse: [Hq, T] float32 (natural log).
 *   - cu_seqlens: DEVICE pointer to B + 1 int32 offsets (4-byte aligned),
 *     cu_seqlens[0] = 0, cu_seqlens[B] = T, non-decreasing; sequence b owns
 *     tokens cu_seqlens[b] .. cu_seqlens[b+1] - 1 and may be empty.
 *   - max_seqlen >= every sequence's length (the grid is sized by it).
 *   - causal keeps key j for query i iff j <= i, positions local to the
 *     sequence; nothing crosses a sequence boundary. GQA as in fa_fwd.
 * The offsets are read on the device, so the host cannot check them: a
 * sequence longer than max_seqlen or offsets outside [0, T] make the kernels
 * skip that sequence and record FA_ERR_INVALID_ARG | (64 << 8) in the device
 * status word (fa_last_device_status). T = 0 or max_seqlen = 0 returns FA_OK
 * without launching. d is 64, 96, 128, 192 or 256 for fa_fwd_varlen and 64, 96
 * or 128 for fa_bwd_varlen.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal, float scale,
                        cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd_varlen needs: D and -LSE log2 e as float32
 * [B * Hq, 128 * ceil(max_seqlen / 128)] and the float32 dQ accumulator
 * [T, Hq, d], each rounded up to 256 bytes. Returns 0 for invalid sizes.
 */
size_t fa_bwd_varlen_workspace_size(int B, int Hq, int Hkv, int total, int max_seqlen, int d);

/*
 * Backward of a packed variable-length batch by recomputation (fa_bwd's
 * method, layouts and conventions of fa_fwd_varlen). `o` and `lse` are
 * fa_fwd_varlen's outputs for the same inputs; dq, dk, dv are overwritten.
 * The workspace is overwritten; its contents on entry do not matter.
 */
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens,
                        void* workspace, size_t workspace_bytes,
                        int B, int Hq, int Hkv, int total, int max_seqlen, int d, int causal, float scale,
                        cudaStream_t stream);

/*
 * Largest scratch, in bytes, that fa_bwd_noalloc can use (32 MiB). A problem
 * fits when fa_bwd_workspace_size(B, Hq, Hkv, N, d) <= FA_BWD_NOALLOC_MAX_BYTES.
 * The scratch holds 8 bytes per query row padded to Npad = 128 * ceil(N / 128)
 * rows per head, plus 4 * d bytes per real query row, so about 64,500 query
 * rows (B * Hq * N) at d = 128 and 127,000 at d = 64 when N is a multiple of
 * 128, and fewer when padding is a large share of N (small or ragged N).
 */
#define FA_BWD_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)

/*
 * Backward pass that needs no workspace from the caller. The pages have no
 * counterpart: this is a convenience of the library, not part of the method.
 * It is fa_bwd with its scratch (D, -LSE log2 e and the fp32 dQ accumulator)
 * taken from a fixed array of FA_BWD_NOALLOC_MAX_BYTES inside the library's
 * device memory, held on every GPU that loads the library until the process
 * exits. It is meant for callers that cannot allocate device memory at the
 * point of the call (C code with no device allocator of its own, or code
 * that must not call cudaMalloc/cudaFree there because they synchronise the
 * device). Arguments, layouts and results are those of fa_bwd.
 *   - Allocates nothing: no cudaMalloc, no cudaFree.
 *   - Argument errors are reported as fa_bwd reports them (null pointer,
 *     invalid size or scale, misalignment, checked in that order); after
 *     them, FA_ERR_WORKSPACE, launching nothing, when fa_bwd_workspace_size
 *     for these sizes exceeds FA_BWD_NOALLOC_MAX_BYTES.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls share the one array. Each call rewrites every scratch value it
 *     reads, so leftovers from earlier calls do not matter, but calls that can
 *     run at the same time on the GPU (other streams, other threads) race and
 *     must be serialised by the caller.
 */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv,
                         int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                         cudaStream_t stream);

/*
 * Bytes of device workspace fa_fwd_fp8 needs: e4m3 copies of Q, K, V
 * (rotated Q and K) and one float32 scale per 64-row block of each. Returns 0
 * for invalid sizes.
 */
size_t fa_fp8_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * FP8 (e4m3) forward with block quantisation and incoherent processing:
 * "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
 * Low-precision" (abstract) names both techniques and gives neither the
 * block shape nor the rotation. Here: Q and K are rotated by
 * diag(sigma) H_d (Sylvester Hadamard, sigma a +-1 vector drawn from
 * `rotation_seed` by SplitMix64, the same for Q and K) when use_rotation is
 * non-zero; Q, K, V are quantised with one float32 scale per 64-row block
 * (s = amax / 448); P is quantised per 128-key tile with V's block scale
 * folded in. Inputs are bf16; O is bf16, LSE float32. Only d = 128 is built,
 * and B * Hq at most 65535 (FA_ERR_UNSUPPORTED otherwise; the same limits
 * hold for fa_fp8_quantize and fa_fwd_fp8_quantized). The workspace is
 * overwritten; afterwards it
 * holds, each region starting on a 1024-byte boundary: e4m3 codes of Q
 * [B*Hq, N, d], K and V [B*Hkv, N, d], then float32 block scales of Q
 * [B*Hq, ceil(N/64)], K and V [B*Hkv, ceil(N/64)].
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                     uint64_t rotation_seed, int use_rotation,
                     void* workspace, size_t workspace_bytes,
                     int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                     cudaStream_t stream);

/*
 * The two halves of fa_fwd_fp8, for callers that quantise once and run the
 * forward several times (a fixed key/value set), or that time the FP8
 * forward apart from its pre-pass. fa_fwd_fp8 is exactly fa_fp8_quantize
 * followed by fa_fwd_fp8_quantized on the same stream.
 *
 * fa_fp8_quantize: rotates (when use_rotation is non-zero) and block-quantises
 * q, k, v (bf16) into `workspace`, in the layout described at fa_fwd_fp8.
 * Same size rules and errors as fa_fwd_fp8.
 */
fa_status fa_fp8_quantize(const void* q, const void* k, const void* v,
                          uint64_t rotation_seed, int use_rotation,
                          void* workspace, size_t workspace_bytes,
                          int B, int Hq, int Hkv, int N, int d, cudaStream_t stream);

/*
 * fa_fwd_fp8_quantized: the FP8 forward from a workspace that
 * fa_fp8_quantize filled for the same B, Hq, Hkv, N, d and use_rotation
 * (the rotation's 1/d is folded into the softmax scale, so use_rotation must
 * match); the workspace is only read. Writes O (bf16) and LSE (float32).
 */
fa_status fa_fwd_fp8_quantized(const void* workspace, size_t workspace_bytes, void* o, float* lse,
                               int use_rotation, int B, int Hq, int Hkv, int N, int d, int causal,
                               float scale, cudaStream_t stream);

/*
 * Bytes of device workspace fa_fwd_mxfp8 needs: e4m3 codes of Q, K, V and
 * their E8M0 exponent bytes (layout at fa_fwd_mxfp8). Returns 0 for invalid
 * sizes and for d != 128.
 */
size_t fa_mxfp8_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * MXFP8 forward: the FP8 forward with the block quantisation that B200's
 * tensor cores apply in hardware. "FlashAttention-3: Fast and Accurate
 * Attention with Asynchrony and Low-precision" (abstract) names block
 * quantisation without fixing the block; here each block is 32 elements
 * along a product's contraction with one power-of-two (E8M0) scale, per the
 * OCP Microscaling Formats (MX) specification v1.0:
 *   Q and K (after the rotation diag(sigma) H_d when use_rotation != 0, as in
 *   fa_fwd_fp8): each row in blocks of 32 columns;
 *   V: each column in blocks of 32 keys;
 *   P: each row of each 96-key tile in blocks of 32 keys.
 * Shared exponent e = floor(log2 amax) - 8 clamped to [-127, 127] (-127 for
 * a zero block), codes e4m3(x 2^-e) with saturation at 448 (scale_rule 0,
 * the specification's); scale_rule 1 takes e + 1 where amax's significand
 * exceeds 1.75, so that no element saturates. Other scale_rule values:
 * FA_ERR_INVALID_ARG. Only d = 128 is built, and B * Hq at most 65535
 * (FA_ERR_UNSUPPORTED otherwise). bf16 q [B, Hq, N, d], k, v [B, Hkv, N, d] and o
 * [B, Hq, N, d], float32 lse [B, Hq, N], all 16-byte aligned and owned by the
 * caller. The workspace (at least fa_mxfp8_workspace_size bytes, 16-byte
 * aligned, else FA_ERR_WORKSPACE / FA_ERR_MISALIGNED) is overwritten; it then
 * holds, each region starting on a 1024-byte boundary: e4m3 codes of Q
 * [B*Hq, N, d], K and V [B*Hkv, N, d]; exponent bytes (e + 127) of Q
 * [B*Hq, N, 4] and K [B*Hkv, N, 4] (one per 32 columns), and of V
 * [B*Hkv, d, nb] with nb = 4 * ceil(N / 96): per column one 4-byte word per
 * 96-key tile (the forward's key tile), bytes 0-2 the exponents of its three
 * 32-key blocks (blocks past N: the exponent of zeros, 0), byte 3 zero.
 */
fa_status fa_fwd_mxfp8(const void* q, const void* k, const void* v, void* o, float* lse,
                       uint64_t rotation_seed, int use_rotation, int scale_rule,
                       void* workspace, size_t workspace_bytes,
                       int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                       cudaStream_t stream);

/*
 * Bytes of device workspace fa_fwd_decode needs for these sizes and
 * num_ctas (0 = automatic, as in fa_fwd_decode): for each CTA of the split
 * pass and each KV head, a float32 partial output row and a float32
 * log-sum-exp per query row. Independent of the device. Returns 0 for invalid
 * or unsupported sizes.
 */
size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas);

/*
 * Forward for few query rows against a long key sequence (decoding with a
 * key/value cache): q, o are [B, Hq, Nq, d] bf16, k, v [B, Hkv, Nk, d] bf16,
 * lse [B, Hq, Nq] float32 (natural log). The computation is fa_fwd's with
 * Nq rows: "FlashAttention: The Algorithm That Made Long-Context AI
 * Possible" (sections "The quadratic bottleneck in standard attention" and
 * "What tiling changes"); the pages do not discuss decoding. With causal
 * non-zero the queries are the last Nq positions of the sequence: query i
 * keeps keys j <= i + Nk - Nq (requires Nk >= Nq).
 * Work split: the (KV head, 64-key tile) pairs are divided evenly among the
 * CTAs of a split pass, each taking a contiguous run; a second kernel merges
 * the partial results of each head by log-sum-exp. num_ctas = 0 runs as many
 * CTAs as fit on the current device at once (at most 1024); a positive value
 * asks for that many (capped at the number of pairs). The result does not
 * depend on the split beyond floating-point rounding.
 * Supported: d = 64 or 128, and (Hq / Hkv) * Nq <= 16 query rows per KV head
 * (FA_ERR_UNSUPPORTED otherwise). causal with Nk < Nq or num_ctas < 0 is
 * FA_ERR_INVALID_ARG. `workspace` is device memory of at least
 * fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_ctas) bytes, 16-byte
 * aligned (FA_ERR_WORKSPACE / FA_ERR_MISALIGNED otherwise); it is
 * overwritten. Two kernels run on `stream`. If a kernel gives up on a bounded
 * wait (FA_ERR_TIMEOUT from fa_last_device_status), o and lse are undefined.
 */
fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                        void* workspace, size_t workspace_bytes,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                        int num_ctas, cudaStream_t stream);

/* Human-readable name of a status code (static storage, never null). */
const char* fa_status_string(fa_status s);

/*
 * Device status word of the current device, then cleared. 0 when no kernel
 * has given up on a bounded wait or met bad packed-batch offsets since the
 * last call. Otherwise the low byte is an fa_status (FA_ERR_TIMEOUT, or
 * FA_ERR_INVALID_ARG for offsets; in the debug library also FA_ERR_BOUNDS)
 * and bits 8.. name the site: the wait that gave up, 64 for the offsets
 * check, 96 + n for bounds check n. Synchronises the device. Returns -1 if
 * the word could not be read.
 */
int fa_last_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_FA_H */
