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
 *  - d is 32, 64, 96, 128, 192 or 256 (32, 96 and 192 run the 64-, 128-
 *    and 256-wide kernels on zero-filled columns; the 256-wide backward runs
 *    two thread blocks per 128-key tile, each owning half of dK, dV and dQ's
 *    columns).  1 <= N <= 2^23; B * H <= 65535 and
 *    B * H * ceil(N / 128) <= 2^31 - 1 (one thread block per head and
 *    128-row tile; the 256-wide backward needs twice that product within the
 *    bound); larger requests return FA_ERR_UNSUPPORTED.
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
 *    keeps no device memory of its own apart from a status word per device
 *    and the fixed 64 MiB array of fa_bwd_noalloc (present on a device once
 *    that module is loaded there: at its first call under CUDA's default lazy
 *    loading, at library load with CUDA_MODULE_LOADING=EAGER).
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
  FA_ERR_UNSUPPORTED = 2, /* valid request the kernels do not cover (d not 32/64/96/128/192/256, sizes too large) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed */
  FA_ERR_TIMEOUT = 4,     /* a kernel gave up on a pipeline wait (reported by fa_last_device_status) */
  FA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than fa_bwd_workspace_size() */
  FA_ERR_BOUNDS = 6       /* only the FA_DEBUG_BOUNDS build: a kernel skipped a global-memory
                             access outside its buffer (reported by fa_last_device_status) */
} fa_status_t;

/* Forward pass.  Writes O (bf16 [B,H,N,d]) and LSE (fp32 [B,H,N]).
 * q, k, v, o, lse: device pointers (see conventions above). */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float softmax_scale, int causal, const int32_t* seqlens,
                   float dropout_p, uint64_t seed, const uint8_t* block_mask, void* stream);

/* Bytes of device workspace fa_bwd needs for these sizes: per (b, h) and per
 * query row rounded up to a multiple of 128, one fp32 -LSE_i * log2(e), one
 * fp32 -D_i = -sum_c dO_ic O_ic and D fp32 dQ accumulators (D = 64 for
 * d <= 64, 128 for d = 96 / 128, 256 for d = 192 / 256).  0 on bad sizes. */
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
 *  fa_bwd_prepare: from o, lse, dout fills the workspace with -D_i, the
 *    negated log2-domain LSE -LSE_i * log2(e) (-inf for rows without keys and
 *    for the padding rows up to the next multiple of 128, so that their P is
 *    exactly 0) and zeroed dQ accumulators.  Reads the softmax statistics the
 *    forward saved.
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
 *    cudaGetSymbolAddress.  Under CUDA's lazy module loading (the default)
 *    that lookup is also when the module holding the array is loaded on the
 *    device, i.e. when its 64 MiB is reserved: make the first call at
 *    start-up, outside any allocator callback and before any stream capture
 *    (or set CUDA_MODULE_LOADING=EAGER to reserve it when the library is
 *    loaded).  The address is cached per device and context and looked up
 *    again after a context teardown such as cudaDeviceReset.
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

/* ------------------------------------------------------------------------
 * General layouts: strided tensors, packed variable-length batches, N_q != N_k
 * ------------------------------------------------------------------------
 * The pages' BERT-large workload is a batch of sequences of different
 * lengths (researchpapers.dev "FlashAttention 详解", section 关键结果); the
 * entry points below take them packed, with no padding rows, as well as
 * token-major ([B, N, H, d]) or any other strided layout whose d is
 * contiguous, different query and key counts, and head dims 32, 64, 96, 128,
 * 192 and 256.
 * The computation is the one above, per batch entry (or packed sequence) b:
 *  - positions i, j are counted inside sequence b (masks, dropout counter);
 *  - causal: query i attends key j iff j <= i + Nk_b - Nq_b, Nq_b / Nk_b the
 *    sequence's query / key counts (bottom-right alignment: the last query
 *    sees every key; rows with no key get O = 0, LSE = -inf); seqlens_k
 *    masks keys j >= seqlens_k[b] without moving this alignment;
 *  - block_mask: device uint8 [ceil(seqlen_q / 128)][ceil(seqlen_k / 128)],
 *    indexed by (i / 128, j / 128), shared by all sequences and heads.
 *
 * Element strides of one tensor viewed as [batch, head, row, d], d contiguous.
 * Every stride must be a non-negative multiple of 8 elements (16 bytes); the
 * batch stride is ignored for the packed layout. */
typedef struct {
  int64_t batch, head, row;
} fa_strides_t;

typedef struct {
  int batch;     /* B: batch entries (padded layout) or packed sequences */
  int heads;     /* H */
  int head_dim;  /* d: 32, 64, 96, 128, 192 or 256 */
  /* Padded layout: rows of every batch entry (queries, keys).  Packed layout:
   * an upper bound of every sequence's query / key count (longer sequences
   * are cut to it). */
  int seqlen_q, seqlen_k;
  /* Packed layout: device int32[B + 1] offsets (0 = cu[0] <= ... <= cu[B]);
   * sequence b's queries are rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 of
   * Q, O, dO, dQ, its keys rows cu_seqlens_k[b] .. of K, V, dK, dV.  Both
   * NULL for the padded layout, both set for the packed one.  Offsets are
   * clamped to [0, total] on the device, so bad offsets give wrong results
   * but never touch memory outside the tensors. */
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  int total_q, total_k; /* packed layout: rows of the packed tensors (>= 1) */
  const int32_t* seqlens_k; /* key padding: device int32[B] or NULL */
  float softmax_scale;
  int causal;
  float dropout_p;
  uint64_t seed;
  const uint8_t* block_mask;
  fa_strides_t q, k, v, o, dout, dq, dk, dv;
  /* Dropout positions: this call's query rows are rows dropout_row0 .. and its
   * keys keys dropout_key0 .. of the sequence the keep bits are keyed by (the
   * call evaluates one block of a longer sequence, as in a context-parallel
   * ring); 0, 0 for a whole sequence.  Both >= 0, dropout_key0 a multiple of
   * 8 (one Philox call covers 8 keys), dropout_row0 + seqlen_q and
   * dropout_key0 + seqlen_k at most 2^31 - 1; otherwise FA_ERR_INVALID_ARG.
   * The masks are not moved: they stay relative to the call's own rows. */
  int64_t dropout_row0, dropout_key0;
  /* Grouped-query attention: K and V (and dK, dV) have heads_kv heads, and
   * query head h reads K / V head h / (heads / heads_kv); heads_kv must divide
   * heads (otherwise FA_ERR_INVALID_ARG), with fewer than 32768 query heads
   * per K / V head (otherwise FA_ERR_UNSUPPORTED).  0, or heads: one K / V
   * head per query head.  dK and dV of a K / V head are the sums over its
   * query heads, deterministic as without grouping (when the backward splits
   * a group over several thread blocks, each writes its own fp32 partial sums
   * and they are added in a fixed order). */
  int heads_kv;
} fa_attention_desc_t;

/* Forward pass for a general layout.  LSE is fp32 [B, H, seqlen_q]
 * contiguous (padded layout) or [H, total_q] (packed layout).  Rows of O and
 * LSE past a sequence's end (padded layout) or that belong to no sequence
 * (packed layout) are not written. */
fa_status_t fa_fwd_ex(const fa_attention_desc_t* desc, const void* q, const void* k,
                      const void* v, void* o, float* lse, void* stream);

/* Workspace bytes of fa_bwd_ex: padded layout B * H * ceil(seqlen_q / 128) * 128
 * rows, packed layout H * (ceil(total_q / 128) * 128 + 256 B) rows, each of
 * 8 + 4 D bytes (D = 64 for d <= 64, 128 for d = 96 / 128, 256 for d = 192 /
 * 256); with grouped K / V heads whose backward units are split into S parts
 * (few units for the SM count), two fp32 dK / dV areas of
 * S * tb * heads_kv * key rows * D elements more (tb = B padded, 1 packed; key
 * rows = seqlen_k padded, total_k packed).  0 if the description is invalid. */
size_t fa_bwd_ex_workspace_size(const fa_attention_desc_t* desc);

/* Backward pass for a general layout (dQ like Q, dK / dV like K / V; the
 * strides of each come from the description).  Same workspace rules as
 * fa_bwd.  dK, dV rows of keys beyond a sequence's key length are 0. */
fa_status_t fa_bwd_ex(const fa_attention_desc_t* desc, const void* q, const void* k,
                      const void* v, const void* o, const float* lse, const void* dout, void* dq,
                      void* dk, void* dv, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Combining partial results (context-parallel attention)
 * ------------------------------------------------------------------------
 * When the keys are split into disjoint blocks that are processed apart (one
 * block per GPU, the blocks passed around a ring), each block b gives a
 * partial (O_b, LSE_b) normalised over its own keys, and the full result is
 * LSE = ln sum_b exp(LSE_b), O = sum_b exp(LSE_b - LSE) O_b: the rescaling
 * of the online softmax across key blocks (suanlizi.com summary, section
 * 分块计算（Tiling）; researchpapers.dev, section 分块与重计算), applied between
 * kernel calls instead of inside one.  The pages name multi-GPU IO-aware
 * attention as the next step (suanlizi.com summary, future-work section on
 * multi-GPU IO optimisation).
 *
 * fa_merge_partial: o_acc (fp32 [rows, d], 16-byte aligned) and lse_acc
 *   (fp32 [rows]) hold the result so far (start: any finite o_acc, lse_acc =
 *   -inf); merges in o_part (bf16 [rows, d], contiguous) with lse_part.
 *   d in {32, 64, 96, 128, 192, 256}.  A part or accumulator with LSE = -inf adds
 *   nothing; both empty gives O = 0, LSE = -inf.
 * fa_accumulate_bf16: acc[i] += part[i] for i < n (fp32 += bf16), n a multiple
 *   of 8, both 16-byte aligned: sums of gradient parts over key / query blocks.
 * fa_convert_f32_bf16: out[i] = bf16(in[i]) (round to nearest even), n a
 *   multiple of 8.
 * All three are asynchronous on `stream` and allocate nothing. */
fa_status_t fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part,
                             const float* lse_part, int64_t rows, int d, void* stream);
fa_status_t fa_accumulate_bf16(float* acc, const void* part, int64_t n, void* stream);
fa_status_t fa_convert_f32_bf16(void* out, const float* in, int64_t n, void* stream);

/* ------------------------------------------------------------------------
 * Fused QKV projection in front of attention
 * ------------------------------------------------------------------------
 * The pages extend IO-awareness to the model's other layers, which all read
 * and write HBM (suanlizi.com summary, section IO-感知优化的普遍性).  This is
 * the layer that feeds attention: with x bf16 [B N, d_model] (token t = b N + n,
 * row-major), w bf16 [3 H d, d_model] (the three projection matrices stacked,
 * as one linear layer stores them) and bias bf16 [3 H d] or NULL,
 *   Y = x w^T + bias (fp32 accumulation, rounded once to bf16),
 *   Q[b, h, n, e] = Y[b N + n, h d + e], K and V from columns H d + ... and
 *   2 H d + ..., each written as bf16 [B, H, N, d] (fa_fwd's layout),
 * with no intermediate [B N, 3 H d] tensor.  d is 64 or 128, H d a multiple of
 * 128, d_model a multiple of 8, B N <= 65535 * 128; all pointers 16-byte
 * aligned device memory owned by the caller.  Asynchronous on `stream`;
 * bounded waits as in the attention kernels. */
fa_status_t fa_qkv_projection(const void* x, const void* w, const void* bias, void* q, void* k,
                              void* v, int B, int N, int H, int d, int d_model, void* stream);

/* Human-readable name of a status code (static storage). */
const char* fa_status_string(fa_status_t status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: FA_OK, or FA_ERR_TIMEOUT if a kernel gave up on a wait
 * since the last call.  FA_ERR_CUDA if the synchronisation itself fails. */
fa_status_t fa_last_device_status(void* stream);

/* Per-wait time limit of the kernels in nanoseconds (default 4e9).  Values
 * below 1e6 are raised to 1e6.  Applies to launches made after the call. */
void fa_set_wait_timeout_ns(uint64_t ns);

/* Test support: enabled = 0 makes the kernels of later launches walk a
 * block mask byte by byte instead of through the per-CTA bitmask they build
 * in shared memory (the walk a mask too long for the bitmask always takes);
 * 1, the default, restores the bitmask.  Both visit the same tiles in the
 * same order, so O, LSE, dK and dV come out identical and dQ equal up to the
 * order of its fp32 reductions. */
void fa_debug_set_block_mask_bitmap(int enabled);

/* Test support: the number of parts a backward unit of grouped K / V heads
 * is split into (each walking that share of the group's query heads and
 * adding its dK / dV into fp32 accumulators).  0, the default, chooses it from
 * the size of the problem; a value that does not divide the group is ignored.
 * Applies to workspace sizes computed and launches made after the call. */
void fa_debug_set_gqa_split(int parts);

/* 1 in the bounds-checking build (FA_DEBUG_BOUNDS: every global-memory access
 * the kernels make outside TMA is checked against its buffer's extent, an
 * out-of-range one skipped and FA_ERR_BOUNDS recorded), 0 otherwise. */
int fa_debug_bounds_checking(void);

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
