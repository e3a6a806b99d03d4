/*
 * vq.h -- C ABI of libvq: B200 (sm_100a) kernels for linear layers whose
 * weights are stored as bit-packed codebook indices (VQ / residual VQ).
 *
 * The method (what the calls compute)
 * -----------------------------------
 * A weight matrix W (out_features N x in_features Kin) is cut, row by row,
 * into vectors of d consecutive input-dimension weights ("VPTQ Guide: Extreme
 * 2-Bit Vector Quantization", section "The Information-Theoretic Superiority
 * of Vector Quantization"; section "Step 2", which slices W.view(-1, v)).
 * Row o has nvec = ceil(Kin / d) vectors; vector j of row o is replaced by a
 * b_m-bit index i_m[o][j] into codebook m, C_m in fp16 [K_m = 2^b_m][d], for
 * one or two codebooks (section "2. Multi-Stage Residual Vector Quantization
 * (RVQ)": w_hat = C1[idx1] + C2[idx2]; "Vector Quantization for LLM Weights in
 * Production", section "2. AQLM: Additive Multi-Codebook Vector Quantization":
 * a sum of M = 1 or 2 centroids).  An optional per-output-row fp16 scale s and
 * bias t complete the layer (section "1. QuIP#": per-channel scaling).  The
 * dequantised weight is
 *
 *     W_hat[o][j*d + e] = fp16( (C1[i1][e] + C2[i2][e]) * s[o] + t[o] )
 *
 * for j*d + e < Kin, each of +, *, + an fp32 operation rounded to nearest even
 * in that order, then one rounding to fp16 (with one codebook the first sum is
 * just C1[i1][e]; a missing scale skips the multiply, a missing bias skips the
 * add).  Components of the last vector past Kin are ignored.  The products are
 * y = x . W_hat^T ("VPTQ Guide", section "Step 3: Fused Low-Bit VPTQ Linear
 * Layer"), computed without writing W_hat to global memory, as the pages
 * describe for production kernels ("Vector Quantization for LLM Weights in
 * Production", section "2. Lookup Table (LUT) Overhead vs. Bit-Shifting":
 * fused lookup and accumulation, no intermediate fp16 global writes).
 *
 * Storage format of the indices (this library's reading; the pages fix only
 * the field width b = log2 K, e.g. "16-bit uint per 8 weights")
 * ---------------------------------------------------------------
 * One stream per codebook, one stream row per output row, rows idx_row_words
 * 32-bit words apart.  Field j of a row occupies bits [j*b, j*b + b), bits
 * numbered least-significant first inside little-endian 32-bit words.  Rows
 * start 16-byte aligned: idx_row_words is a multiple of 4 and at least
 * ceil(nvec*b / 128) * 4.  Bits past nvec*b in a row are ignored.  Indices are
 * unsigned and K = 2^b exactly, so every index is inside its codebook.
 *
 * A second storage order, VQ_IDX_TILE4 (also this library's), holds the same
 * fields tiled by four vectors: a book's stream is ceil(nvec/4) tiles,
 * idx_row_words 32-bit words apart; tile t covers vectors 4t..4t+3, and inside
 * it the rows follow one another, row o contributing one 4b-bit record with
 * the fields of vectors 4t, 4t+1, 4t+2, 4t+3 in that order.  Field (o, j)
 * thus occupies bits [(4*o + j%4)*b, +b) of tile j/4, numbered as above.
 * Tiles start 16-byte aligned: idx_row_words is a multiple of 4 and at least
 * ceil(N*4*b / 128) * 4.  Fields of vectors >= nvec are ignored.  It costs
 * the same bits per weight; the decode lookup-table kernel (vq_gemv, batch 1)
 * needs it, because one tile row puts four consecutive vectors of a row next
 * to those of the following rows.  vq_repack_tile4 converts a row-order
 * layer.
 *
 * Conventions for every call
 * --------------------------
 * - Pointers named "device" must be CUDA device (or managed) memory visible
 *   to the current device; the caller allocates and owns them.  The library
 *   keeps no allocation between calls (it caches per-device attributes only).
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *   default stream).  Argument errors are detected on the host and returned
 *   before anything is launched; nothing is written then.
 * - Launch failures return VQ_ERR_CUDA; vq_last_cuda_error() gives the
 *   cudaError_t.  Kernels never trap.  Kernels that wait on the device (an
 *   mbarrier of a TMA / tensor-core pipeline) bound every wait: after about
 *   2 s (VQ_WAIT_BUDGET in the environment sets the budget in SM clocks) the
 *   kernel records VQ_ERR_TIMEOUT in the status word of its workspace (see
 *   each call), lets its copies in flight land, and returns.
 * - fp16 / bf16 values are passed as their 16-bit patterns.
 * - All calls are thread-safe; concurrent calls on different streams may not
 *   share an output or a workspace buffer.
 */
#ifndef VQ_H_
#define VQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VQ_ABI_VERSION 4

#if defined(__GNUC__)
#define VQ_API __attribute__((visibility("default")))
#else
#define VQ_API
#endif

typedef enum vq_status {
    VQ_OK = 0,
    VQ_ERR_INVALID_ARG = 1,   /* a size, pointer or field is out of range       */
    VQ_ERR_UNSUPPORTED = 2,   /* well-formed, but outside what is implemented   */
    VQ_ERR_ALIGNMENT = 3,     /* a pointer or leading dimension is misaligned   */
    VQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required     */
    VQ_ERR_CUDA = 5,          /* a CUDA call or kernel launch failed            */
    VQ_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up (status word) */
} vq_status;

typedef enum vq_idx_layout {
    VQ_IDX_ROWS = 0,          /* one stream row per output row (default)        */
    VQ_IDX_TILE4 = 1          /* tiles of four vectors, rows consecutive inside */
} vq_idx_layout;

typedef enum vq_dtype {
    VQ_BF16 = 0,
    VQ_FP16 = 1,
    VQ_FP32 = 2
} vq_dtype;

/*
 * One quantised layer.  All pointers are device pointers.
 *   out_features   N >= 0
 *   in_features    Kin >= 0 (need not be a multiple of vec_dim)
 *   vec_dim        d, 1..16
 *   n_books        1 or 2 (main codebook plus optional residual/additive one)
 *   log2k[m]       b_m, 1..16; K_m = 2^b_m
 *   idx[m]         packed stream of book m, 16-byte aligned: [N][idx_row_words[m]]
 *                  uint32 in row order, [ceil(nvec/4)][idx_row_words[m]] tiled
 *   idx_row_words[m]  stride between stream rows (row order) or tiles (tiled
 *                  order) in 32-bit words, a multiple of 4, >= ceil(nvec*b_m /
 *                  128) * 4 in row order, >= ceil(N*4*b_m / 128) * 4 tiled
 *   codebook[m]    fp16 [K_m][d] row-major, 16-byte aligned, finite values
 *   scale          fp16 [N], or NULL for no scale
 *   bias           fp16 [N], or NULL for no bias
 *   idx_layout     VQ_IDX_ROWS or VQ_IDX_TILE4 (a zero-filled struct means rows)
 *   reserved       must be 0
 *   out_bias       fp16 [N], or NULL: the output-side bias of the product,
 *                  y[b][o] = sum_k x[b][k] W_hat[o][k] + out_bias[o], added in
 *                  fp32 to the accumulated product before y is rounded to its
 *                  type.  The layer's forward ends in F.linear(x, W_hat, bias)
 *                  ("VPTQ Guide", section "Step 3: Fused Low-Bit VPTQ Linear
 *                  Layer"); this is that bias, distinct from the per-row bias
 *                  t above, which is part of W_hat.  vq_dequant ignores it.
 *                  (Added in ABI version 4, which made the struct 104 bytes.)
 * Entries for m >= n_books are ignored.
 */
typedef struct vq_layer_desc {
    int32_t out_features;
    int32_t in_features;
    int32_t vec_dim;
    int32_t n_books;
    int32_t log2k[2];
    const uint32_t* idx[2];
    int64_t idx_row_words[2];
    const uint16_t* codebook[2];
    const uint16_t* scale;
    const uint16_t* bias;
    int32_t idx_layout;
    int32_t reserved;
    const uint16_t* out_bias;
} vq_layer_desc;

/*
 * vq_dequant -- write W_hat (fp16 [N][ldw], device) exactly as defined above:
 * bit-exact with the fixed-order fp32 definition.  Columns >= Kin of each row
 * are not written.  ldw >= Kin.  Follows "VPTQ Guide", section "Step 2"
 * (ResidualVectorQuantizer.dequantize) with the scale and bias of the layer.
 * Errors: VQ_ERR_INVALID_ARG (bad layer, NULL w_hat with N*Kin > 0, ldw < Kin),
 * VQ_ERR_ALIGNMENT (misaligned idx/codebook), VQ_ERR_CUDA.
 */
VQ_API vq_status vq_dequant(const vq_layer_desc* layer, uint16_t* w_hat, int64_t ldw, void* stream);

/*
 * vq_repack_tile4 -- write the index streams of a row-order layer in the
 * tiled order (VQ_IDX_TILE4), on the device.  src->idx_layout must be
 * VQ_IDX_ROWS.  For each book m < src->n_books, dst[m] (device, 16-byte
 * aligned, caller-owned, not overlapping src->idx[m]) receives
 * ceil(nvec/4) * dst_tile_words[m] words, every one of them written: fields,
 * then zero padding (also for vectors >= nvec).  dst_tile_words[m] follows the
 * tiled-order rule above.  A layer description that points idx[] at dst[],
 * with idx_row_words = dst_tile_words and idx_layout = VQ_IDX_TILE4, then
 * describes the same weights.
 * Errors: VQ_ERR_INVALID_ARG (bad layer or tile stride, NULL dst with data,
 * src already tiled), VQ_ERR_ALIGNMENT, VQ_ERR_CUDA.
 */
VQ_API vq_status vq_repack_tile4(const vq_layer_desc* src, uint32_t* const dst[2],
                                 const int64_t dst_tile_words[2], void* stream);

/*
 * vq_gemv_workspace_size -- bytes of device workspace vq_gemv needs for this
 * layer and batch (0 when it needs none).  Host-only; launches nothing.
 */
VQ_API vq_status vq_gemv_workspace_size(const vq_layer_desc* layer, int32_t batch, size_t* bytes);

/*
 * vq_gemv -- decode-time product y[b][o] = sum_k x[b][k] * W_hat[o][k] for
 * b < batch (1..16), fp32 accumulation, without materialising W_hat.  The
 * pages place this regime at B = 1 to 8, memory-bandwidth bound
 * ("Vector Quantization for LLM Weights in Production", section "1. Prefill
 * vs. Decode Bottlenecks"); the fused lookup-and-accumulate kernel is the one
 * "VPTQ Guide", section "Step 3", describes.
 *   x        device, x_dtype (VQ_BF16 or VQ_FP16) [batch][ldx], ldx >= Kin
 *   y        device, y_dtype (VQ_BF16, VQ_FP16 or VQ_FP32) [batch][ldy], ldy >= N
 *   workspace  device scratch of at least vq_gemv_workspace_size() bytes
 *            (may be NULL when that size is 0), 256-byte aligned; its contents
 *            on entry do not matter
 * Scale and bias are applied as y = s[o] * sum_k x[k] (C1+C2)[o][k]
 * + t[o] * sum_k x[k], equal to the definition up to the fp16 rounding of
 * W_hat (well inside a 2e-3 normwise relative error).
 * Tiled layers (VQ_IDX_TILE4) with batch 1, one book, vec_dim 8, 16-bit
 * indices and N <= 65536 run the lookup-table kernel: per group of four
 * vectors it forms the dot products of x with every centroid (fp32 products
 * of fp16 operands on the tensor cores, each group of x scaled by a power of
 * two so that no product can overflow fp16), rounds them to fp16, and sums the
 * entries the indices select.  That rounding adds about 2^-12 relative error
 * per term, inside the same tolerance as long as the codebook's values are
 * normal fp16 numbers (|c| >= 2^-14).  Books of up to 2^12 entries (one or
 * two, d = 6 or 8) get a table kernel without slices.  Tiled layers run one
 * table pass per row of x up to batch 2 (2^16 book), 3 (small books, rows of
 * at most 1024 vectors) or 5 (small books, longer rows).
 * Larger batches (from 2 in row order) of layers with one 2^16-entry d = 8
 * book, or with books of up to 2^12 + 2^12 entries and d = 6 or 8 (from 3 in
 * row order), run the tensor-core kernels: per 128 rows of W and step of
 * eight vectors, the centroids (the sum of both books' centroids, rounded
 * once to fp16) are gathered into a shared-memory tile and multiplied on the
 * tcgen05 tensor cores with x, each row of x scaled by a power of two into
 * fp16 (exact products, fp32 accumulation); values of a row below 2^-29 of
 * its largest lose precision as fp16 subnormals.  The first 32-bit word of
 * their workspace is a status word: VQ_OK, or VQ_ERR_TIMEOUT if a bounded
 * device-side wait gave up (readable after the stream completes).  Every
 * other case runs the split-K gather kernel, which reads either index order.
 * The environment variables VQ_LUT_MAX_BATCH (0 turns the table kernels
 * off), VQ_TC_MIN_BATCH and VQ_TCS_MIN_BATCH (above 16 turns the 2^16-book or
 * the small-book tensor-core kernel off) move those limits, for
 * measurements.
 * Errors: VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED (batch > 16), VQ_ERR_ALIGNMENT
 * (x or y not aligned to its element size), VQ_ERR_WORKSPACE, VQ_ERR_CUDA.
 */
VQ_API vq_status vq_gemv(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t batch,
                  int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * vq_gemv_noalloc -- vq_gemv for callers that cannot allocate device memory
 * where they run the layer (a serving loop working inside a pre-reserved pool,
 * a plug-in called from another framework's allocator-controlled context, or
 * code with no CUDA allocation API at hand).  The pages have no counterpart:
 * this is a deployment convenience of this library.  Same arguments and
 * results as vq_gemv, minus the workspace: the split-K scratch comes from a
 * fixed device array of VQ_NOALLOC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits.  The call
 * allocates nothing (no cudaMalloc, no allocating library routine).
 *   - Plans whose scratch can shrink run within the array (the table kernels'
 *     per-block row sums: fewer blocks); a plan that needs more scratch than
 *     VQ_NOALLOC_SCRATCH_BYTES and cannot shrink (split-K partial sums) makes
 *     the call return VQ_ERR_WORKSPACE.  vq_gemv_workspace_size() reports the
 *     unconstrained plan, so a size above the array does not by itself mean
 *     that this call fails.
 *   - The array and the plan belong to the current device: `stream` must be a
 *     stream of the current device (or NULL), else VQ_ERR_INVALID_ARG.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - All calls on a device share the array; calls whose kernels overlap on
 *     the GPU (e.g. on two streams at once) race on it and must be ordered by
 *     the caller.  No part of the array needs to start at zero, so its
 *     contents from an earlier call do not matter.
 */
#define VQ_NOALLOC_SCRATCH_BYTES (8u << 20)
VQ_API vq_status vq_gemv_noalloc(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype,
                                 int32_t batch, int64_t ldx, void* y, vq_dtype y_dtype,
                                 int64_t ldy, void* stream);

/*
 * vq_gemv_multi -- y_l = x . W_hat_l^T for n_layers (1..16) layers that read
 * the same x (the projections of one transformer block: gate and up, or q, k
 * and v), with the same meaning, arguments and errors as n_layers calls of
 * vq_gemv (y[l] and ldy[l] per layer).  At batch 1, two to four tiled layers
 * that all have one 2^16-entry d = 8 book, or all have a 2^12-entry main book
 * with the same residual (d = 6 with 2^4, or d = 8 with 2^8), and whose rows
 * fit eight 8192-row batches (a power of two per layer), run as one
 * lookup-table launch over all their tasks and one reduction launch, which
 * fills the machine better than separate calls
 * ("VQ in Production", section "1. Prefill vs. Decode Bottlenecks": decode
 * is a sequence of small, memory-bound products).  Every other case runs the
 * layers one after another on the stream.
 */
VQ_API vq_status vq_gemv_multi_workspace_size(const vq_layer_desc* const* layers, int32_t n_layers,
                                              int32_t batch, size_t* bytes);
VQ_API vq_status vq_gemv_multi(const vq_layer_desc* const* layers, int32_t n_layers, const void* x,
                               vq_dtype x_dtype, int32_t batch, int64_t ldx, void* const* y,
                               vq_dtype y_dtype, const int64_t* ldy, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * vq_gemm_workspace_size -- bytes of device workspace vq_gemm needs for this
 * layer, row count m and activation type.  Host-only.
 */
VQ_API vq_status vq_gemm_workspace_size(const vq_layer_desc* layer, int32_t m, vq_dtype x_dtype,
                                 size_t* bytes);

/*
 * vq_gemm -- prefill product y[i][o] = sum_k x[i][k] * W_hat[o][k] for
 * i < m, on the tcgen05 tensor cores (fp16 x fp16 products, fp32 accumulation
 * in tensor memory).  W_hat tiles are either produced on chip from the index
 * streams (fused form: W_hat never reaches global memory) or written once into
 * the workspace by the vq_dequant kernel and streamed in by TMA (staged form);
 * the call picks the form from the codebook sizes and m, and tiled layers
 * (VQ_IDX_TILE4) always take the staged form.  The pages call prefill the
 * compute-bound regime where lookups compete with the matrix multiply
 * ("Vector Quantization for LLM Weights in Production", section "1. Prefill
 * vs. Decode Bottlenecks", and the "GEMV / Tensor Core Dot Products" stage of
 * its dequantisation diagram).
 *   x        device, x_dtype (VQ_BF16 or VQ_FP16) [m][ldx]; 16-byte aligned,
 *            ldx a multiple of 8, ldx >= Kin.  bf16 activations become fp16
 *            operands row by row, each row scaled by a power of two that puts
 *            its largest magnitude in [2^14, 2^15) and undone in the epilogue:
 *            any finite bf16 value is accepted, and values above 2^-29 of
 *            their row's largest are exact (smaller ones lose precision as
 *            fp16 subnormals).  fp16 activations are used as given.
 *   y        device, y_dtype [m][ldy]; ldy >= N
 *   workspace  device scratch of at least vq_gemm_workspace_size() bytes,
 *            256-byte aligned; its first 32-bit word is a status word (VQ_OK,
 *            or VQ_ERR_TIMEOUT if a bounded device-side wait gave up),
 *            readable after the stream completes
 * Scale and bias are applied in the epilogue as for vq_gemv.
 * Errors: as vq_gemv; VQ_ERR_UNSUPPORTED for vec_dim > 8 or m > 2^30.
 */
VQ_API vq_status vq_gemm(const vq_layer_desc* layer, const void* x, vq_dtype x_dtype, int32_t m,
                  int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Nearest-centroid encoder: the step that produces the index streams.
 *
 * Vector j of output row o is v = W[o][j*d .. j*d+d) (the same orientation as
 * the layer format); the last vector of a row keeps only its in_features -
 * j*d valid components when in_features is not a multiple of d, and the
 * distance below then runs over those components only.  For book 1,
 *     idx_1[o][j] = argmin_k sum_e (v_e - C_1[k][e])^2,
 * ties to the lowest k, the distance taken exactly as in fp64 (each
 * difference, square and running sum rounded once, components in order).
 * With two books the second index encodes the residual of the first (the
 * greedy cascade): v_e - C_1[idx_1][e], formed in fp64, against C_2.
 * Follows "VPTQ Guide: Extreme 2-Bit Vector Quantization", section "The
 * Information-Theoretic Superiority of Vector Quantization" (q = argmin_k
 * ||w - c_k||^2) and section "2. Multi-Stage Residual Vector Quantization
 * (RVQ)" (the second stage quantises what the first leaves).
 *
 * Method: the tensor cores evaluate ||c||^2 - 2<v, c> for 128 vectors x 256
 * centroids per tcgen05 MMA (fp16 operands scaled by one power of two per
 * book, fp32 accumulation in tensor memory) and the epilogue keeps each
 * vector's two smallest values.  Where the gap between them exceeds twice a
 * bound on the arithmetic error, the smallest is the exact argmin; every
 * other vector (and every partial last vector) is decided by an fp64 pass
 * over the whole book.  The result therefore equals the exact definition.
 *
 * Hessian-weighted form (h != NULL): the distance becomes
 *     D_H(v, c) = (v - c)^T H_v (v - c),
 * H_v the sub-matrix of the layer's Hessian h on the vector's channels
 * (rows and columns j*d .. j*d+d-1, fewer for a partial last vector), for
 * both stages of the cascade ("VPTQ Guide", section "1. Second-Order
 * Hessian-Weighted Optimization": D_H(w, c_k) = (w - c_k)^T H_Iv (w - c_k);
 * the page writes the residual stage unweighted, which is the case H = I).
 * Exactly as in fp64: t_e = v_e - c_e, g_e = sum_f H[e][f] t_f (f ascending),
 * D = sum_e t_e g_e (e ascending), every operation rounded once, ties to the
 * lowest k.  Method: per vector z = H_s v (H_s = (H + H^T) / 2) is split
 * into two fp16 halves for the tensor cores, which give -2<z, c>; the
 * epilogue adds c^T H_v c, precomputed per (block of channels, centroid) in
 * the workspace; near ties and partial last vectors take the fp64 pass as
 * above.  vec_dim must be <= 8.  h is typically vq_hessian's output.
 *
 *   out_features, in_features   N, Kin >= 0
 *   vec_dim        d, 1..14
 *   n_books        1 or 2;  log2k[m] in 1..16
 *   w, ldw         device fp16 [N][ldw], ldw >= Kin, finite values
 *   codebook[m]    device fp16 [K_m][d], finite values
 *   idx[m], idx_row_words[m]   device output streams in row order (the layer
 *                  format above): 16-byte aligned, idx_row_words[m] a multiple
 *                  of 4 and >= ceil(nvec*b_m/128)*4; every word of the N rows
 *                  is written (fields, then zero padding)
 *   h, ldh         NULL for the plain distance, or device fp32 [Kin][ldh],
 *                  ldh >= Kin, 4-byte aligned, finite values (read only on
 *                  the diagonal blocks); ABI version 4
 */
typedef struct vq_encode_desc {
    int32_t out_features;
    int32_t in_features;
    int32_t vec_dim;
    int32_t n_books;
    int32_t log2k[2];
    const uint16_t* w;
    int64_t ldw;
    const uint16_t* codebook[2];
    uint32_t* idx[2];
    int64_t idx_row_words[2];
    const float* h;
    int64_t ldh;
} vq_encode_desc;

/* Bytes of device workspace vq_encode needs (host-only, launches nothing;
 * only the sizes and strides of desc are read). */
VQ_API vq_status vq_encode_workspace_size(const vq_encode_desc* desc, size_t* bytes);

/*
 * vq_encode -- run the encoder above on `stream`.  workspace: device,
 * 256-byte aligned, at least vq_encode_workspace_size() bytes; its first
 * 32-bit word is a status word (VQ_OK, or VQ_ERR_TIMEOUT if a bounded
 * device-side wait gave up), readable after the stream completes.
 * Errors: VQ_ERR_INVALID_ARG (sizes, NULL pointers with data, short strides),
 * VQ_ERR_UNSUPPORTED (vec_dim > 8 with h), VQ_ERR_ALIGNMENT,
 * VQ_ERR_WORKSPACE, VQ_ERR_CUDA.
 */
VQ_API vq_status vq_encode(const vq_encode_desc* desc, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * Randomized Hadamard transform (QuIP#-style incoherence processing): a layer
 * may be quantised in a rotated basis, W~ = U W V^T with U, V orthogonal
 * randomized Walsh-Hadamard matrices, so that y = W x = U^T (W~ (V x))
 * ("Vector Quantization for LLM Weights in Production", section "1. QuIP#:
 * Incoherence Processing and Lattice Codebooks"; "Sub-4-Bit Quantization",
 * section "QuIP#: Incoherence Processing": Hadamard plus random signs).
 * A row of length n is transformed in blocks of b = the largest power of two
 * dividing n (at most 2^15), i.e. by (I (x) H_b) diag(s) / sqrt(b):
 *   forward:  out[k b + i] = b^-1/2 sum_j H_b[i][j] s[k b + j] in[k b + j]
 *   inverse:  out[k b + j] = s[k b + j] b^-1/2 sum_i H_b[j][i] in[k b + i]
 * H_b[i][j] = (-1)^popcount(i & j) (Sylvester), s[t] = -1 where bit t of
 * `signs` is set (32-bit words, LSB first; ceil(n / 32) words), else +1.
 * Arithmetic in fp32 (fast Walsh-Hadamard butterflies in shared memory).
 */

/* vq_rht -- transform `rows` (<= 65535) rows of length n: in [rows][ld_in] of
 * in_dtype, out [rows][ld_out] of out_dtype (bf16, fp16 or fp32), device
 * pointers, inverse = 0 for V, 1 for V^T.  in and out may not overlap.
 * Errors: VQ_ERR_INVALID_ARG, VQ_ERR_UNSUPPORTED (rows > 65535),
 * VQ_ERR_ALIGNMENT, VQ_ERR_CUDA. */
VQ_API vq_status vq_rht(const void* in, vq_dtype in_dtype, int32_t rows, int32_t n, int64_t ld_in,
                        const uint32_t* signs, int32_t inverse, void* out, vq_dtype out_dtype,
                        int64_t ld_out, void* stream);

/* vq_gemv_rht -- y = U^T (W~ (V x)) for a layer whose streams encode W~:
 * V x with signs_in (in_features bits), the product as vq_gemv with x~ in
 * fp16 and y~ in fp32, then U^T with signs_out (out_features bits).  Same
 * arguments and errors as vq_gemv; the workspace (vq_gemv_rht_workspace_size,
 * 256-byte aligned) also holds x~ and y~. */
VQ_API vq_status vq_gemv_rht_workspace_size(const vq_layer_desc* layer, int32_t batch, size_t* bytes);
VQ_API vq_status vq_gemv_rht(const vq_layer_desc* layer, const uint32_t* signs_in,
                             const uint32_t* signs_out, const void* x, vq_dtype x_dtype,
                             int32_t batch, int64_t ldx, void* y, vq_dtype y_dtype, int64_t ldy,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * vq_hessian -- the normalised, damped Hessian of a layer's inputs ("VPTQ
 * Guide", section "Step 1: Hessian Matrix Collection"; section "1.
 * Second-Order Hessian-Weighted Optimization": H = 2 X X^T over the tokens):
 *   h = 2 X^T X / n_tokens,  h[i][i] += 0.01 * mean_i h[i][i]
 * X: device, x_dtype (VQ_BF16 or VQ_FP16) [n_tokens][ldx], d_in columns
 * used; h: device fp32 [d_in][ldh].  X^T X runs on the tcgen05 tensor cores
 * (bf16 or fp16 operands as given, exact products, fp32 accumulation); the
 * normalisation and damping in fp64, rounded once to fp32.  The workspace
 * (vq_hessian_workspace_size, 256-byte aligned) holds X^T and a status word
 * (first 32 bits: VQ_OK or VQ_ERR_TIMEOUT).
 * Errors: VQ_ERR_INVALID_ARG (n_tokens < 1, short strides, NULL buffers),
 * VQ_ERR_ALIGNMENT, VQ_ERR_WORKSPACE, VQ_ERR_CUDA.
 */
VQ_API vq_status vq_hessian_workspace_size(int32_t n_tokens, int32_t d_in, size_t* bytes);
VQ_API vq_status vq_hessian(const void* x, vq_dtype x_dtype, int32_t n_tokens, int32_t d_in, int64_t ldx,
                            float* h, int64_t ldh, void* workspace, size_t workspace_bytes, void* stream);

/* Static description of a status code (never NULL). */
VQ_API const char* vq_status_string(vq_status status);

/* The cudaError_t of the last VQ_ERR_CUDA returned on this host thread. */
VQ_API int vq_last_cuda_error(void);

/* VQ_ABI_VERSION of the loaded library. */
VQ_API int vq_abi_version(void);

/* Host-only: number of CUDA kernels this library has launched in this process
 * (all threads, all devices).  Lets a caller count the device work behind a
 * sequence of calls. */
VQ_API uint64_t vq_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* VQ_H_ */
