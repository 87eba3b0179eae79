/*
 * fp8q.h — C ABI of libfp8q: the FP8 data-movement hot path of FP8-Flow-MoE on one
 * B200 (sm_100a).
 *
 *   row-wise 1x128 E4M3 quantization with power-of-two (UE8M0) scales
 *   -> scaling-aware direct transpose to the column-wise (1x128 along tokens) layout,
 * plus the in-library naive dequant->transpose->requant baseline and the fused
 * SwiGLU+quantize and permute+pad+quantize neighbours.
 *
 * Sources (page title, section):
 *   "FP8-Flow-MoE: A Casting-Free FP8 Recipe without Double Quantization Error
 *    (MLSys 2026)" review: 核心方法 (scaling-aware transpose; fused permute+padding;
 *    fused SwiGLU+quantization), 关键观察 2, 问题与动机 (the naive three-pass path).
 *   "01 · DeepSeek FP8 与 DeepGEMM：Hopper 软件方案": §1 (wgrad reduces over tokens),
 *    §3 (1x128 activation tiles, SF [T, C/128], online amax), §5.6 (M-grouped
 *    contiguous expert layout), §8 (UE8M0 scales).
 *   "低精度（Low Precision）：从 FP8 到 FP4 的训练与推理" §2 (E4M3: max 448, no Inf).
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers on the current CUDA device, allocated and owned by
 *     the caller; the library never allocates, frees or retains them.  Each must be
 *     16-byte aligned and address a contiguous row-major array.
 *   - E4M3 codes are bytes (OCP E4M3FN: bias 7, max 448, no Inf).  Scales are UE8M0
 *     bytes: S = 2^(byte - 127).  An all-zero tile has scale byte 127 (S = 1).
 *   - Each call is asynchronous on `stream` (NULL = the legacy default stream) and
 *     returns after the launch.  Its kernels are launched as programmatic dependent
 *     launches: their thread blocks may be placed on the GPU while the previous kernel
 *     in the stream is finishing, but none touches memory before that kernel has
 *     completed, so stream order holds as for a plain launch; a later kernel launched
 *     the same way may likewise be placed early.  Host-detectable argument errors
 *     return before any launch and leave every output untouched.  Errors that only the
 *     device can see (bad group offsets, routing indices out of range, a bounded wait
 *     that expired) are recorded in one per-device status word; read it with
 *     fp8q_last_device_status().
 *   - Inputs must be finite (no NaN/Inf); codes given to the transposes must come from
 *     a quantization (never 0x7F/0xFF).
 *   - Calls that share an output buffer and overlap on the GPU race; order them on one
 *     stream.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so that users need no CUDA header. */
typedef struct CUstream_st *fp8q_stream_t;

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_NULL = 1,    /* a required pointer is NULL */
    FP8Q_ERR_SHAPE = 2,   /* sizes violate the layout rules (multiples of 128, groups) */
    FP8Q_ERR_ALIGN = 3,   /* a pointer is not 16-byte aligned */
    FP8Q_ERR_ARG = 4,     /* other invalid argument (workspace too small, capacity, ...) */
    FP8Q_ERR_CUDA = 5,    /* a CUDA runtime/driver call failed (launch, attribute query) */
    FP8Q_ERR_TIMEOUT = 6, /* device: a bounded wait on an mbarrier expired */
    FP8Q_ERR_DEVICE = 7   /* device: invalid data seen by a kernel (e.g. expert index) */
} fp8q_status;

/* Static, NUL-terminated description of a status code. */
const char *fp8q_status_string(fp8q_status s);

/* Synchronizes `stream`, then reads and clears the current device's status word.
 * Returns FP8Q_OK if no kernel recorded an error since the last read, the first
 * recorded device error otherwise, or FP8Q_ERR_CUDA if the synchronization failed. */
fp8q_status fp8q_last_device_status(fp8q_stream_t stream);

/* Row-wise 1x128 quantization (DeepSeek FP8 §3; FP8-Flow-MoE 关键观察 2).
 *   x  : bf16 [rows, cols], cols % 128 == 0, rows >= 0.
 *   q  : u8   [rows, cols]      out: E4M3 codes, q = RNE(x / S) saturating at 448.
 *   sf : u8   [rows, cols/128]  out: UE8M0 byte e + 127 of tile (t, j), where
 *        e = ceil(log2(amax/448)) (the smallest e with amax <= 448 * 2^e), e = 0 for
 *        an all-zero tile, clamped to [-127, 127].
 * rows == 0 is a no-op.  Errors: NULL, ALIGN, SHAPE (cols % 128 != 0, negatives),
 * CUDA. */
fp8q_status fp8q_quantize_rowwise(const void *x, int64_t rows, int64_t cols, uint8_t *q, uint8_t *sf,
                                  fp8q_stream_t stream);

/* Scaling-aware direct transpose (FP8-Flow-MoE 核心方法).  For every 128x128 block
 * (row block b, column block j): e_max = max of the block's 128 row-tile exponents;
 * each row t shifts its codes by k_t = e_max - e_t >= 0, q' = RNE_e4m3(decode(q)*2^-k_t)
 * (an exponent-field subtract, the mantissa re-rounded only when the result turns
 * subnormal); the block is written transposed with scale byte e_max + 127 for each of
 * its 128 channels.
 *   q, sf : the row-wise pair from fp8q_quantize_rowwise, [rows, cols], [rows, cols/128].
 *   group_offsets : NULL for one dense group (then rows % 128 == 0), or a DEVICE
 *        int32 array [num_groups + 1] with offsets[0] == 0, non-decreasing, every
 *        group size a multiple of 128, offsets[num_groups] <= rows (rows is then the
 *        capacity of q).  Violations found on the device set FP8Q_ERR_SHAPE in the
 *        status word and skip the offending blocks.
 *   qt  : u8 out.  Dense: [cols, rows].  Grouped: group g (M_g = off[g+1]-off[g] rows)
 *         is the row-major array [cols, M_g] starting at byte cols*off[g].
 *   sft : u8 out.  Dense: [cols, rows/128].  Grouped: group g is [cols, M_g/128]
 *         starting at byte cols*off[g]/128.
 * Bytes past the last group are not written.  Errors: NULL, ALIGN, SHAPE, ARG
 * (num_groups < 1), CUDA. */
fp8q_status fp8q_direct_transpose(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                                  const int32_t *group_offsets, int32_t num_groups, uint8_t *qt,
                                  uint8_t *sft, fp8q_stream_t stream);

/* Bytes of device workspace fp8q_naive_transpose needs: 4 * rows * cols (a BF16
 * dequantized copy and its BF16 transpose). */
size_t fp8q_naive_workspace_bytes(int64_t rows, int64_t cols);

/* Naive baseline that the direct transpose replaces (FP8-Flow-MoE 问题与动机 and
 * 核心方法, the three-pass conversion): (1) dequantize each code to BF16,
 * v = bf16(decode(q) * 2^e); (2) transpose v; (3) requantize every 128-token column
 * tile with a fresh power-of-two scale by the rule of fp8q_quantize_rowwise.
 * Three kernel launches.  Same arguments, layouts and errors as fp8q_direct_transpose,
 * plus a caller-owned device workspace of at least fp8q_naive_workspace_bytes(rows,
 * cols) bytes, 16-byte aligned (ERR_ARG if smaller). */
fp8q_status fp8q_naive_transpose(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                                 const int32_t *group_offsets, int32_t num_groups, uint8_t *qt,
                                 uint8_t *sft, void *workspace, size_t workspace_bytes,
                                 fp8q_stream_t stream);

/* Fused SwiGLU + quantization (FP8-Flow-MoE 核心方法: the activation is produced
 * directly as FP8).  y = silu(gate) * up in fp32 with silu(g) = g / (1 + exp(-g)),
 * every operation one IEEE fp32 rounding and exp the library's Cody-Waite/Taylor
 * evaluation; then the row-wise quantization of y, and, if qt != NULL, the direct
 * transpose of that result in the same kernel.
 *   gate, up : bf16 [rows, cols], cols % 128 == 0.
 *   q, sf    : out, as fp8q_quantize_rowwise.
 *   qt, sft  : out, [cols, rows] and [cols, rows/128], or both NULL to skip; when given,
 *              rows % 128 == 0.
 * The first call on a device evaluates the spec's silu values once and keeps them in
 * the library's static device memory (31 KB); later calls copy them from there.
 * Errors: NULL, ALIGN, SHAPE, ARG (only one of qt/sft given), CUDA. */
fp8q_status fp8q_swiglu_quant(const void *gate, const void *up, int64_t rows, int64_t cols, uint8_t *q,
                              uint8_t *sf, uint8_t *qt, uint8_t *sft, fp8q_stream_t stream);

/* Bytes of device workspace fp8q_permute_pad_quant needs; 0 for arguments no permute
 * accepts (negative tokens, topk < 1, num_experts < 1, tokens*topk beyond 2^31 - 1). */
size_t fp8q_permute_workspace_bytes(int64_t tokens, int32_t topk, int32_t num_experts);

/* Fused permute + pad + row-wise quantize (FP8-Flow-MoE 核心方法: Fused
 * Permute+Padding; DeepSeek FP8 §5.6: M-grouped contiguous expert rows).
 *   x        : bf16 [tokens, hidden], hidden % 128 == 0.
 *   topk_idx : int32 [tokens, topk], expert ids in [0, num_experts).
 *   Expert e receives the pairs (t, s) with topk_idx[t, s] == e, in (t, s) row-major
 *   order; its segment is padded with zero rows to a multiple of `align`.
 *   q, sf    : out [max_out_rows, hidden], [max_out_rows, hidden/128]; row r of the
 *              segment of pair (t, s) holds the row-wise quantization of x[t]; padding
 *              rows hold codes 0x00 and scale byte 127; rows at or beyond
 *              expert_offsets[num_experts] are not written.
 *   max_out_rows : capacity, >= tokens*topk + num_experts*(align-1).
 *   expert_offsets : out int32 [num_experts + 1], exclusive scan of padded sizes.
 *   row_id_map     : out int32 [tokens*topk], destination row of pair (t, s).
 *   workspace      : device, >= fp8q_permute_workspace_bytes(...), 16-byte aligned.
 *   align in [1, 4096]; num_experts in [1, 4096]; topk in [1, 64]; tokens*topk and
 *   max_out_rows at most 2^31 - 1 (row ids are int32), else FP8Q_ERR_SHAPE / ARG.
 * An expert id out of range sets FP8Q_ERR_DEVICE in the status word (outputs are
 * then unspecified).  Errors: NULL, ALIGN, SHAPE, ARG, CUDA. */
fp8q_status fp8q_permute_pad_quant(const void *x, int64_t tokens, int64_t hidden, const int32_t *topk_idx,
                                   int32_t topk, int32_t num_experts, int32_t align, uint8_t *q,
                                   uint8_t *sf, int64_t max_out_rows, int32_t *expert_offsets,
                                   int32_t *row_id_map, void *workspace, size_t workspace_bytes,
                                   fp8q_stream_t stream);

/* Options of fp8q_quantize_rowwise_colwise (bit flags). */
#define FP8Q_ZERO_TILE_MIN_SCALE 0x1u /* all-zero tiles take e = -127 (byte 0x00), not e = 0 */
#define FP8Q_SF_PACKED_UE8M0 0x2u     /* scales as packed UE8M0 words (see below) */

/* Bytes of a packed UE8M0 scale tensor for an FP8 operand with `mn` rows along M/N and
 * `k` elements along K (k % 128 == 0): 4 * ceil(k/512) * (mn rounded up to 4).
 * 0 for non-positive sizes. */
size_t fp8q_packed_sf_bytes(int64_t mn, int64_t k);

/* Single-pass quantization into both layouts: one read of X produces the row-wise
 * (Q, SF) of fp8q_quantize_rowwise and the column-wise (Q^T, SF^T) that
 * fp8q_direct_transpose would make from them - byte for byte the same results
 * (FP8-Flow-MoE 核心方法; DeepSeek FP8 §1, §3).  Moves 4 bytes per element instead of
 * the 5 of the two separate calls.
 *   x   : bf16 [rows, cols], cols % 128 == 0; rows % 128 == 0 when qt is given.
 *   q   : u8 [rows, cols]   out, as fp8q_quantize_rowwise.
 *   sf  : out. Unpacked: u8 [rows, cols/128].  Packed: u32 [ceil(cols/512), rows4].
 *   qt  : u8 [cols, rows] out, or NULL for the row-wise layout only.
 *   sft : out, NULL iff qt is NULL.  Unpacked: u8 [cols, rows/128] (as the direct
 *         transpose).  Packed: u32 [ceil(rows/512), cols].
 *   flags: FP8Q_ZERO_TILE_MIN_SCALE - an all-zero 1x128 tile gets e = -127 instead of
 *         e = 0, so it never raises Smax of its 128x128 block (its codes are +-0 either
 *         way; a fully zero block gets SF^T byte 0).  Off, results equal
 *         fp8q_quantize_rowwise + fp8q_direct_transpose exactly.
 *         FP8Q_SF_PACKED_UE8M0 - scales as packed UE8M0 (DeepSeek FP8 §8: the SM100 GEMM
 *         reads four power-of-two scales per int32): word (g, m) at index g*mn4 + m
 *         (mn4 = mn rounded up to 4; MN-major) holds the scale bytes of the K tiles
 *         4g..4g+3 of row m in bits 0-7, 8-15, 16-23, 24-31.  Bytes of K tiles past the
 *         last, and words of the padding rows m >= mn, are 0.  sf/sft must then be
 *         4-byte aligned and hold fp8q_packed_sf_bytes(rows, cols) and
 *         fp8q_packed_sf_bytes(cols, rows) bytes.
 * x, q and qt must be 16-byte aligned.  Errors: NULL, ALIGN, SHAPE, ARG (unknown flag
 * bits, qt/sft not both NULL or both set), CUDA. */
fp8q_status fp8q_quantize_rowwise_colwise(const void *x, int64_t rows, int64_t cols, uint32_t flags,
                                          uint8_t *q, void *sf, uint8_t *qt, void *sft,
                                          fp8q_stream_t stream);

/* Fused unpermute + unpad: the combine side of the expert path (FP8-Flow-MoE 核心方法,
 * fused Unpermute+Unpadding).  Each token gathers its K expert rows back and sums them
 * with its routing weights; padding rows are never read:
 *   out[t, h] = BF16_RNE( fma chain over s = 0..K-1 of w[t,s] * v(row_id_map[t,s], h) ),
 * acc starting at -0 (so one slot gives its product exactly, sign of zero included),
 * one fp32 fused multiply-add per slot in slot order, where v is the fp32 value of the
 * row element (this order is the library's reading; the pages fix none).
 *   y          : BF16 [rows, hidden] when y_sf is NULL, else E4M3 codes u8 [rows, hidden]
 *                with y_sf u8 [rows, hidden/128] row-wise UE8M0 scales (v = decode(q) *
 *                2^(byte - 127), exact unless it overflows fp32).  hidden % 128 == 0.
 *   rows       : rows of y (the permuted buffer's capacity).
 *   row_id_map : int32 [tokens, topk], as written by fp8q_permute_pad_quant.  An entry
 *                outside [0, rows) sets FP8Q_ERR_DEVICE in the status word and its slot
 *                is skipped.
 *   weights    : fp32 [tokens, topk] routing weights, or NULL for all ones (the
 *                backward of the permute: the sum of a token's K row gradients).
 *   out        : BF16 [tokens, hidden].
 * Results must be finite (NaN outputs are unspecified).  y and out 16-byte aligned;
 * row_id_map and weights 4-byte aligned.  Errors: NULL, ALIGN, SHAPE, ARG (topk not in
 * [1, 64]), CUDA. */
fp8q_status fp8q_unpermute_unpad(const void *y, const uint8_t *y_sf, int64_t rows, int64_t hidden,
                                 const int32_t *row_id_map, const float *weights, int64_t tokens,
                                 int32_t topk, void *out, fp8q_stream_t stream);

/* FP8-input permute + pad: the pages' FP8 dataflow quantizes before the dispatch, so the
 * permute receives row-wise codes and scales (FP8-Flow-MoE 核心方法 and casting-free
 * dataflow).  Same routing, offsets, row ids, padding rows and errors as
 * fp8q_permute_pad_quant; the payload of a destination row is the token's codes and
 * scale bytes, copied:
 *   xq  : u8 [tokens, hidden] E4M3 codes, 16-byte aligned;
 *   xsf : u8 [tokens, hidden/128] UE8M0 scale bytes.
 * All other arguments and the workspace (fp8q_permute_workspace_bytes) as in
 * fp8q_permute_pad_quant.  Permuting quantize_rowwise(X) this way gives byte for byte
 * what fp8q_permute_pad_quant(X) gives. */
fp8q_status fp8q_permute_pad_fp8(const uint8_t *xq, const uint8_t *xsf, int64_t tokens, int64_t hidden,
                                 const int32_t *topk_idx, int32_t topk, int32_t num_experts, int32_t align,
                                 uint8_t *q, uint8_t *sf, int64_t max_out_rows, int32_t *expert_offsets,
                                 int32_t *row_id_map, void *workspace, size_t workspace_bytes,
                                 fp8q_stream_t stream);

/* The path at MX granularity (low-precision format table: MXFP8 = E4M3 elements with one
 * power-of-two scale per 32 elements; FP8-Flow-MoE 局限与 Future Work 2: the
 * scaling-aware conversion carried to MX formats).  Same scale rule and shift as above,
 * with 1x32 scaling tiles and 32x32 transpose blocks.
 *   fp8q_quantize_rowwise_mx32: x bf16 [rows, cols], cols % 32 == 0 -> q u8 [rows, cols],
 *     sf u8 [rows, cols/32].  x and q 16-byte aligned.
 *   fp8q_direct_transpose_mx32: (q, sf) as above -> qt u8 [cols, rows], sft u8
 *     [cols, rows/32] holding, for channel h and token group g, the largest scale byte of
 *     the 32x32 block (g, h/32).  This build's kernel needs rows % 128 == 0 and
 *     cols % 128 == 0 (its CTA tile is 128x128, sixteen MX blocks), and rows at most
 *     65535 * 128 (its grid has one row of CTAs per 128 rows).  q and qt 16-byte
 *     aligned, sf and sft 4-byte aligned.
 * Errors: NULL, ALIGN, SHAPE, CUDA. */
fp8q_status fp8q_quantize_rowwise_mx32(const void *x, int64_t rows, int64_t cols, uint8_t *q, uint8_t *sf,
                                       fp8q_stream_t stream);
fp8q_status fp8q_direct_transpose_mx32(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t cols,
                                       uint8_t *qt, uint8_t *sft, fp8q_stream_t stream);

/* ------------------------------------------------------------------ expert-parallel dispatch
 * FP8-Flow-MoE review, 核心方法 (the dispatch moves row-wise FP8 codes together with
 * their scale metadata) and Table 1 (an FP8 all-to-all against BF16: about 1.6x, 1.4x
 * with one Q/DQ pair); DeepSeek FP8 §5.6 (each rank's experts read contiguous row
 * groups).  W ranks hold `experts_per_rank` experts each; global expert e lives on rank
 * e / experts_per_rank as its local expert e % experts_per_rank.
 *
 * Send side, fp8q_ep_dispatch_pack (one source rank): every token goes once to each
 * rank that holds at least one of its top-k experts, carrying its codes, its scale bytes
 * and its k slot ids re-expressed for that rank (the local expert id, or -1 where the
 * slot's expert lives on another rank).
 *   xq, xsf   : u8 [tokens, hidden] codes (16-byte aligned), [tokens, hidden/128] scales.
 *   topk_idx  : int32 [tokens, topk], global expert ids in [0, num_ranks*experts_per_rank).
 *   send_q, send_sf, send_ids : out [max_send_rows, hidden], [.., hidden/128], int32
 *               [.., topk]; rows grouped by destination rank, tokens in order within a
 *               group.  max_send_rows >= tokens * min(num_ranks, topk).
 *   send_offsets : out int32 [num_ranks + 1]: rank d's rows are send_offsets[d] ..
 *               send_offsets[d+1]-1 (these are the all-to-all's send splits).
 *   send_map  : out int32 [tokens, num_ranks]: the send row of (token, rank), or -1.
 *   workspace : device, >= fp8q_ep_pack_workspace_bytes(tokens, num_ranks), 16-aligned.
 *   num_ranks in [1, FP8Q_EP_MAX_RANKS]; topk in [1, 64]; experts_per_rank in [1, 4096].
 *   An expert id out of range sets FP8Q_ERR_DEVICE in the status word (its slot is
 *   then not sent).  Errors: NULL, ALIGN, SHAPE, ARG, CUDA.
 *
 * Receive side, fp8q_ep_recv_permute_fp8 (one destination rank): the rows every source
 * rank sent here, read where they lie (a segment of an all-to-all receive buffer, or any
 * memory this device can address), permuted straight into the expert-grouped, padded
 * layout of fp8q_permute_pad_fp8 for the local experts.  The received rows are numbered
 * in source order (sources[0]'s rows first); slot (r, s) with id e >= 0 goes to local
 * expert e in (r, s) row-major order; each expert's segment is padded with zero rows
 * (codes 0x00, scale byte 127) to a multiple of `align`; a slot with id -1 gets row id
 * -1.  With a single source holding every token and every id local, the result is
 * fp8q_permute_pad_fp8's.
 *   sources   : host array of num_sources segments {q, sf, ids, rows}: codes u8
 *               [rows, hidden] (16-byte aligned), scales u8 [rows, hidden/128], slot
 *               ids int32 [rows, topk] in [-1, experts_per_rank); read during the call
 *               only.  Pointers may be NULL where rows == 0.
 *   q, sf, max_out_rows, expert_offsets [experts_per_rank + 1]: as fp8q_permute_pad_fp8,
 *               with max_out_rows >= R*topk + experts_per_rank*(align-1), R = total rows.
 *   row_id_map: out int32 [R * topk].
 *   workspace : device, >= fp8q_ep_recv_workspace_bytes(R, topk, experts_per_rank).
 *   num_sources in [1, FP8Q_EP_MAX_RANKS]; R*topk <= 2^31 - 1.  An id outside
 *   [-1, experts_per_rank) sets FP8Q_ERR_DEVICE.  Errors: NULL, ALIGN, SHAPE, ARG, CUDA. */
#define FP8Q_EP_MAX_RANKS 64
typedef struct fp8q_ep_source {
  const uint8_t *q;
  const uint8_t *sf;
  const int32_t *ids;
  int64_t rows;
} fp8q_ep_source;
size_t fp8q_ep_pack_workspace_bytes(int64_t tokens, int32_t num_ranks);
fp8q_status fp8q_ep_dispatch_pack(const uint8_t *xq, const uint8_t *xsf, int64_t tokens, int64_t hidden,
                                  const int32_t *topk_idx, int32_t topk, int32_t num_ranks, int32_t experts_per_rank,
                                  uint8_t *send_q, uint8_t *send_sf, int32_t *send_ids, int64_t max_send_rows,
                                  int32_t *send_offsets, int32_t *send_map, void *workspace, size_t workspace_bytes,
                                  fp8q_stream_t stream);
size_t fp8q_ep_recv_workspace_bytes(int64_t rows, int32_t topk, int32_t experts_per_rank);
fp8q_status fp8q_ep_recv_permute_fp8(const fp8q_ep_source *sources, int32_t num_sources, int64_t hidden,
                                     int32_t topk, int32_t experts_per_rank, int32_t align, uint8_t *q, uint8_t *sf,
                                     int64_t max_out_rows, int32_t *expert_offsets, int32_t *row_id_map,
                                     void *workspace, size_t workspace_bytes, fp8q_stream_t stream);

/* Size of the library's static scratch for fp8q_permute_pad_quant_noalloc (4 MiB). */
#define FP8Q_NOALLOC_SCRATCH_BYTES (4u << 20)

/* fp8q_permute_pad_quant for callers that cannot allocate device memory (the paper has
 * no counterpart: this is a deployment convenience).  Some callers cannot call
 * cudaMalloc where they route tokens: their device memory belongs to an allocator they
 * cannot reach from this point, or they run under a fixed, pre-planned memory budget, or
 * they are a plugin handed only its input and output buffers.  This entry point takes
 * the same arguments as fp8q_permute_pad_quant minus the workspace, and keeps the
 * routing scratch in a file-scope device array of FP8Q_NOALLOC_SCRATCH_BYTES instead.
 * It allocates nothing and calls no allocating routine.
 *   Limit: fp8q_permute_workspace_bytes(tokens, topk, num_experts) must not exceed
 *   FP8Q_NOALLOC_SCRATCH_BYTES (about tokens*topk*num_experts/128 bytes; e.g. 2M
 *   token-slot pairs with 256 experts, or 16M with 32); larger requests return
 *   FP8Q_ERR_ARG before any CUDA call.
 *   Memory: every GPU that loads the library holds the array until the process exits.
 *   Set-up: every call looks the array's device address up for the current device
 *   and context (cudaGetSymbolAddress, a host-side lookup once the library's device
 *   code is loaded), so a device reset or another context on the same device gets its
 *   own copy's address.  The first call on a device loads that code: make it before
 *   capturing a stream.
 *   Sharing: all calls on a device use the same array, which keeps the previous call's
 *   contents (nothing in it needs to start at zero: every word is written before it is
 *   read).  Calls that overlap on the GPU (other streams, other threads) race on it:
 *   order them on one stream.
 * Other arguments, results and errors: as fp8q_permute_pad_quant. */
fp8q_status fp8q_permute_pad_quant_noalloc(const void *x, int64_t tokens, int64_t hidden,
                                           const int32_t *topk_idx, int32_t topk, int32_t num_experts,
                                           int32_t align, uint8_t *q, uint8_t *sf, int64_t max_out_rows,
                                           int32_t *expert_offsets, int32_t *row_id_map, fp8q_stream_t stream);

/* Test hook for the bounded-wait machinery (no counterpart on the pages): launches one
 * CTA that waits on an mbarrier nobody arrives at, giving up after `timeout_ns`
 * nanoseconds (clamped to [1e3, 2e9]); the kernel then records FP8Q_ERR_TIMEOUT in the
 * status word and returns normally.  No fault, no trap: the context stays usable. */
fp8q_status fp8q_debug_expire_wait(uint64_t timeout_ns, fp8q_stream_t stream);

/* Test hooks for cross-checks against a CPU implementation (no counterpart on the pages).
 *   fp8q_debug_e4m3_encode_range: out[i] = the E4M3 code (round to nearest even,
 *     saturating to +-448) that every kernel's fp32 -> E4M3 conversion gives for the fp32
 *     with bit pattern first_bits + i, i < n (first_bits + n <= 2^32).
 *   fp8q_debug_exp_spec_range: out[i] = the SwiGLU spec's exp (fp32) of the fp32 with bit
 *     pattern first_bits + i.
 *   fp8q_debug_swiglu_spec: y[i] = silu(gate[i]) * up[i] by the SwiGLU spec, fp32 in and
 *     out (the value fp8q_swiglu_quant quantizes).
 *   fp8q_debug_silu_bf16: y[i] = silu(gate[i]) for n BF16 gate values (n even, gate
 *     4-byte and y 8-byte aligned), computed the way fp8q_swiglu_quant computes it (the
 *     spec's values tabulated in shared memory, from the device's published copy once
 *     one exists, looked up, closed forms outside the table's range).
 * Device pointers; float arrays 4-byte aligned.  Errors: ARG, NULL, ALIGN, CUDA. */
fp8q_status fp8q_debug_e4m3_encode_range(uint32_t first_bits, int64_t n, uint8_t *out, fp8q_stream_t stream);
fp8q_status fp8q_debug_exp_spec_range(uint32_t first_bits, int64_t n, float *out, fp8q_stream_t stream);
fp8q_status fp8q_debug_swiglu_spec(const float *gate, const float *up, int64_t n, float *y, fp8q_stream_t stream);
fp8q_status fp8q_debug_silu_bf16(const void *gate, int64_t n, float *y, fp8q_stream_t stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fp8q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
