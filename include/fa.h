/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention library.
 *
 * The operation is exact softmax attention computed FlashAttention-style: the
 * inputs are tiled through on-chip memory, an online softmax keeps a running
 * row maximum m and row sum l, the N x N score and probability matrices never
 * reach device memory, and the forward pass saves the per-row log-sum-exp
 * LSE = m + ln(l) so that the backward pass can rebuild the probabilities
 * instead of storing them.  Sources for each piece of the definition:
 *   - exactness: the output equals standard attention, only memory traffic
 *     differs (researchpapers.dev "FlashAttention 详解:IO 感知精确注意力,提速
 *     2-4 倍", sections "快速答案" and FAQ "精确的还是近似的");
 *   - tiling + online softmax with rescaling per block (same page, section
 *     "分块与重计算"; suanlizi.com FlashAttention summary, section
 *     "分块计算（Tiling）");
 *   - recomputation in the backward from saved softmax statistics (suanlizi.com
 *     summary, section "重计算"; researchpapers.dev, section "分块与重计算");
 *   - safe softmax with the row maximum subtracted (llm-deploy
 *     tensorrt-llm/flash-attention.md, section on overflow / underflow);
 *   - block-sparse variant that computes only selected blocks (suanlizi.com
 *     summary, section "块稀疏注意力");
 *   - mask and dropout fused into the same kernel (suanlizi.com summary,
 *     description of Figure 1, right).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors Q, K, V, O, dO, dQ, dK, dV are bf16, contiguous [B, H, N, d]
 *    (row-major, d fastest), in device memory, 16-byte aligned.
 *  - LSE is fp32 [B, H, N], natural logarithm; a row with no valid key has
 *    LSE = -inf and O = 0.
 *  - d is 64 or 128.  1 <= N <= 2^23; B * H <= 65535 and
 *    B * H * ceil(N / 128) <= 2^31 - 1 (one thread block per head and
 *    128-row tile); larger requests return FA_ERR_UNSUPPORTED.
 *  - softmax_scale multiplies Q K^T before masking (typically 1/sqrt(d)).
 *  - causal != 0: query i attends key j only if j <= i.
 *  - seqlens: NULL, or device int32[B]; keys j >= seqlens[b] are masked for
 *    batch entry b (values are clamped to [0, N]).  Query rows are not masked.
 *  - dropout_p in [0, 1): inverted dropout on the normalised probabilities.
 *    Keep bit of (b, h, i, j): Philox4x32-10 with key (seed & 0xffffffff,
 *    seed >> 32) and counter (j >> 3, i, h, b); key j takes the 16-bit half
 *    (j & 1) (0 = low) of output word ((j >> 1) & 3) and is kept iff that
 *    value >= t = min(floor(dropout_p * 2^16), 2^16 - 1).  The drop
 *    probability in force is t / 2^16 (0.0999908 for 0.1) and kept values are
 *    divided by 1 - t / 2^16.  dropout_p == 0 draws no random numbers.
 *  - block_mask: NULL, or device uint8[nb][nb] with nb = ceil(N / 128),
 *    shared by all (b, h); entry [r][c] == 0 masks every (query, key) pair with
 *    i / 128 == r and j / 128 == c, and such blocks are neither loaded nor
 *    computed.
 *  - All masks combine by logical AND.
 *  - stream: a cudaStream_t (NULL = the legacy default stream).  Every call is
 *    asynchronous on that stream; nothing is synchronised and nothing printed.
 *  - Ownership: the caller allocates and frees every buffer.  The library
 *    keeps no device memory of its own apart from a status word per device.
 *  - Errors: arguments are validated before any launch; a failed check
 *    returns FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED and launches nothing.
 *    A failed launch returns FA_ERR_CUDA.  A kernel whose internal pipeline
 *    wait exceeds its time limit stops, records FA_ERR_TIMEOUT in the device
 *    status word and returns; fa_last_device_status() reports it.
 */
#ifndef IO_AWARE_EXACT_20_B200_FA_H
#define IO_AWARE_EXACT_20_B200_FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer, p out of range */
  FA_ERR_UNSUPPORTED = 2, /* valid request the kernels do not cover (d not 64/128, sizes too large) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed */
  FA_ERR_TIMEOUT = 4,     /* a kernel gave up on a pipeline wait (reported by fa_last_device_status) */
  FA_ERR_WORKSPACE = 5    /* workspace missing or smaller than fa_bwd_workspace_size() */
} fa_status_t;

/* Forward pass.  Writes O (bf16 [B,H,N,d]) and LSE (fp32 [B,H,N]).
 * q, k, v, o, lse: device pointers (see conventions above). */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float softmax_scale, int causal, const int32_t* seqlens,
                   float dropout_p, uint64_t seed, const uint8_t* block_mask, void* stream);

/* Bytes of device workspace fa_bwd needs for these sizes: per (b, h) and per
 * query row rounded up to a multiple of 128, one fp32 log2-domain LSE, one
 * fp32 D_i = sum_c dO_ic O_ic and d fp32 dQ accumulators.  0 on bad sizes. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/* Backward pass.  Given the forward inputs, its outputs o and lse, and dout
 * (bf16 [B,H,N,d]), writes dq, dk, dv (bf16 [B,H,N,d]).  The masks, scale,
 * dropout_p and seed must be those of the forward call.  workspace: device
 * memory of at least fa_bwd_workspace_size(B,H,N,d) bytes, 256-byte aligned,
 * owned by the caller; its contents on entry do not matter and it may be
 * reused once the call has completed on the stream.  dq is reduced with fp32
 * atomics, so its last bits may vary between runs; dk and dv are deterministic. */
fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float softmax_scale, int causal, const int32_t* seqlens, float dropout_p,
                   uint64_t seed, const uint8_t* block_mask, void* workspace,
                   size_t workspace_bytes, void* stream);

/* The three launches fa_bwd makes, exposed so that each can be timed or
 * scheduled on its own.  Called in this order on one stream with the same
 * workspace they are exactly fa_bwd.
 *  fa_bwd_prepare: from o, lse, dout fills the workspace with D_i, the
 *    log2-domain LSE (+inf where a row has no key, so its P is 0) and zeroed
 *    dQ accumulators.  Reads the softmax statistics the forward saved.
 *  fa_bwd_main: recomputes P block by block from those statistics (the
 *    recomputation of the pages) and writes dk, dv (bf16) and the fp32 dQ
 *    accumulators in the workspace.
 *  fa_bwd_finish: dq = bf16(softmax_scale * accumulator). */
fa_status_t fa_bwd_prepare(const void* o, const float* lse, const void* dout, int B, int H, int N,
                           int d, void* workspace, size_t workspace_bytes, void* stream);
fa_status_t fa_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dk,
                        void* dv, int B, int H, int N, int d, float softmax_scale, int causal,
                        const int32_t* seqlens, float dropout_p, uint64_t seed,
                        const uint8_t* block_mask, void* workspace, size_t workspace_bytes,
                        void* stream);
fa_status_t fa_bwd_finish(void* dq, int B, int H, int N, int d, float softmax_scale,
                          const void* workspace, size_t workspace_bytes, void* stream);

/* Backward pass that allocates nothing (no counterpart in the paper: an
 * interface convenience of this library).  For callers that cannot allocate
 * device memory, for example code inside an allocator or memory-pool callback
 * that must not re-enter the allocator, or a host application that reserves
 * all device memory up front: same arguments and results as fa_bwd without
 * the workspace, which instead lives in a fixed 64 MiB device array inside
 * the library (held on every device that loads it until the process exits).
 *  - Returns FA_ERR_WORKSPACE, launching nothing, when
 *    fa_bwd_workspace_size(B,H,N,d) exceeds 64 MiB (67108864 bytes).
 *  - The first call on a device looks the array's address up with
 *    cudaGetSymbolAddress; make that first call before any stream capture.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents; each call rewrites everything that must start at zero before
 *    using it.  Calls whose kernels overlap on the GPU (unordered streams)
 *    race on the array: issue them on one stream or otherwise serialise them.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine. */
fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                           const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                           int H, int N, int d, float softmax_scale, int causal,
                           const int32_t* seqlens, float dropout_p, uint64_t seed,
                           const uint8_t* block_mask, void* stream);

/* Human-readable name of a status code (static storage). */
const char* fa_status_string(fa_status_t status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: FA_OK, or FA_ERR_TIMEOUT if a kernel gave up on a wait
 * since the last call.  FA_ERR_CUDA if the synchronisation itself fails. */
fa_status_t fa_last_device_status(void* stream);

/* Per-wait time limit of the kernels in nanoseconds (default 4e9).  Values
 * below 1e6 are raised to 1e6.  Applies to launches made after the call. */
void fa_set_wait_timeout_ns(uint64_t ns);

/* Test support: writes the dropout keep bits (1 = kept) of every (b,h,i,j)
 * into keep (device uint8 [B,H,N,N]) using the same device generator as the
 * attention kernels. */
fa_status_t fa_debug_dropout_mask(uint8_t* keep, int B, int H, int N, float dropout_p,
                                  uint64_t seed, void* stream);

/* Test support for the bounded waits: launches one CTA that waits on a
 * pipeline barrier nothing ever signals, so the wait must give up after the
 * configured time limit and record FA_ERR_TIMEOUT (read it with
 * fa_last_device_status).  Faults nothing and leaves the context usable. */
fa_status_t fa_debug_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* IO_AWARE_EXACT_20_B200_FA_H */
