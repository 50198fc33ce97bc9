/*
 * fa.h -- C ABI of the B200 (sm_100a) fused attention library libfa_b200.so.
 *
 * The operation is masked softmax attention with an optional position bias,
 *
 *     out = Softmax(Q K^T * scale + atten_mask + pse) V,
 *
 * as stated by the FlashAttentionScore fusion-operator guide ("operator
 * mathematics", sec. 2, and the call npu_fusion_attention(query, key, value,
 * head_num, input_layout, pse, padding_mask, atten_mask, scale, keep_prob) of
 * its sec. 3.1 with the parameter table of sec. 3.2).  The N x N score matrix
 * is never written to memory: it is built tile by tile with an online softmax
 * (same guide, sec. 2), and the backward pass recomputes the probabilities
 * from the per-row log-sum-exp saved by the forward.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller.  The library never allocates device memory and keeps no state
 *    between calls, except one device-side status word (fa_sync_status)
 *    and the persistent forward's work counters.  Device addresses of these
 *    are looked up once per device, so cudaDeviceReset is not supported
 *    while the library is in use.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call that launches work is asynchronous on that stream.
 *  - Argument errors are detected on the host before anything is launched
 *    and returned synchronously; nothing is written in that case.
 *  - A failed launch returns FA_ERR_CUDA.  Errors inside a running kernel
 *    (a bounded wait that gave up) are recorded in the status word and
 *    reported by fa_sync_status.
 *  - Layouts (input_layout of the guide, sec. 3.2):
 *      FA_LAYOUT_BNSD: q is [B][N][Sq][D], k and v are [B][N][Sk][D].
 *      FA_LAYOUT_BSH : q is [B][Sq][H], k and v are [B][Sk][H] with
 *                      H = N * D and head h at columns h*D .. h*D+D-1.
 *    All contiguous, D innermost.  out, dq, dk, dv use the layout and dtype
 *    of q, k, v (FA_E4M3: out is bf16).  lse is always fp32 [B][N][Sq].
 *  - Dtypes: FA_BF16 or FA_F16 (tensor-core path, D in {64, 128}), or FA_F32
 *    (fp32 FMA path, 1 <= D <= 128).  Accumulation is fp32 in all three; P
 *    and dS enter the tensor core in the operand type.
 *  - FA_E4M3 (forward only, D = 128; the multimodal page's experimental
 *    "pure fp8"): q, k, v are fp8 e4m3 (OCP E4M3, finite range +-448); the
 *    tensor core computes S = Q K^T and O = P V in kind::f8f6f4 with fp32
 *    accumulation, P rounded to e4m3 before P V.  Per-tensor dequantisation
 *    factors are the caller's: fold those of q and k into `scale`, and
 *    multiply the bf16 out by that of v.  fa_bwd returns FA_ERR_UNSUPPORTED.
 *  - Tensor pointers must be 16-byte aligned.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* malformed argument (null, shape, stride)      */
  FA_ERR_UNSUPPORTED = 2,  /* well-formed but not implemented (keep_prob<1) */
  FA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed          */
  FA_ERR_TIMEOUT = 4,      /* a kernel's bounded wait gave up               */
  FA_ERR_CONCURRENT = 5    /* more forward calls ran on one GPU at the same
                              time than the library has work counters (64):
                              the results of the calls involved are invalid */
} fa_status;

typedef enum { FA_LAYOUT_BNSD = 0, FA_LAYOUT_BSH = 1 } fa_layout;
typedef enum { FA_F32 = 0, FA_BF16 = 1, FA_F16 = 2, FA_E4M3 = 3 } fa_dtype;

/* Mask rules (bit flags, combinable).  A key j is visible to query i when
 * every active rule allows it.  Disallowed scores are -inf before the
 * softmax (masked_fill with -inf of the multimodal FlashAttention page,
 * layer 2).  A row with no visible key returns out = 0 and lse = -inf, and
 * contributes nothing to the gradients. */
enum {
  FA_MASK_CAUSAL = 1,      /* j <= i, top-left aligned (the lower-triangular
                              tril mask of the CogVLM page, "attention mask
                              mechanism")                                    */
  FA_MASK_KV_PADDING = 2,  /* j < kv_len[b] (key-side document padding mask,
                              retrieval page, layer 2 SemanticModeler)       */
  FA_MASK_BOOL = 4,        /* mask[b,h,i,j] != 0, 1 = may attend (polarity of
                              create_cross_modal_mask, multimodal page)      */
  FA_MASK_MODALITY = 8     /* allow[id_i][id_j] || (allow_diag && i == j),
                              ids = modality_ids[b][*] in {0, 1}; the
                              cross-modal rule of the multimodal page as a
                              2x2 table, evaluated on the fly (Sq == Sk)    */
};

/* Granularity of the optional tile map (rows x keys of one tile). */
enum { FA_TILE_M = 128, FA_TILE_N = 128 };

typedef struct {
  uint32_t flags;               /* OR of FA_MASK_*                           */
  const int32_t* kv_len;        /* [B] device, FA_MASK_KV_PADDING            */
  const uint8_t* mask;          /* device, FA_MASK_BOOL; element (b,h,i,j) at
                                   b*stride_b + h*stride_h + i*stride_q + j;
                                   a zero stride broadcasts that axis.  With
                                   the pointer and all strides multiples of
                                   16 bytes the forward reads rows 16 bytes
                                   at a time (otherwise byte by byte: the
                                   same result, slower)                      */
  int64_t mask_stride_b, mask_stride_h, mask_stride_q;
  const uint8_t* tile_map;      /* optional, from fa_build_mask_tile_map for
                                   this very mask and shape: lets the kernels
                                   skip tiles with no visible key.  NULL =
                                   treat every tile as partially visible.    */
  const int32_t* modality_ids;  /* [B][S] device, FA_MASK_MODALITY          */
  uint8_t allow[2][2];          /* allow[id_q][id_k], FA_MASK_MODALITY      */
  uint8_t allow_diag;           /* also allow i == j, FA_MASK_MODALITY      */
} fa_mask;

/* Position bias `pse` (guide, sec. 3.2: "optional, supports fusing position
 * encodings such as ALiBi").  `kind` is a bit set; each term is added to the
 * scaled score and is not multiplied by `scale`:
 *   FA_PSE_ALIBI adds -slopes[h] * |i - j|;
 *   FA_PSE_DENSE adds a dense fp32 term A[b][h][i][j] -- the general pse
 *     tensor of sec. 3.2, or a float attention mask added to the scaled
 *     scores as in the guide's unfused steps (sec. 4 step 1).  Element
 *     (b, h, i, j) is read at bias[b*bias_stride_b + h*bias_stride_h +
 *     i*bias_stride_q + j] (strides in elements; 0 broadcasts over b or h,
 *     and bias_stride_q >= Sk is required).  Values are finite or -inf: a
 *     pair whose score is -inf is masked, and a row left with no finite
 *     score gives out = 0, lse = -inf, as with the bool mask.  The array is
 *     read, never written; 16-byte alignment of `bias` and strides that are
 *     multiples of 4 take the vectorised loads (any 4-byte aligned array is
 *     accepted).  FA_PSE_ALIBI | FA_PSE_DENSE adds both. */
enum { FA_PSE_NONE = 0, FA_PSE_ALIBI = 1, FA_PSE_DENSE = 2 };
typedef struct {
  int kind;                     /* FA_PSE_* bit set                          */
  const float* slopes;          /* [N] device, FA_PSE_ALIBI                  */
  const float* bias;            /* device fp32, FA_PSE_DENSE                 */
  int64_t bias_stride_b, bias_stride_h, bias_stride_q;
} fa_pse;

/* Dropout (guide, sec. 3.1/3.2: keep_prob, "Dropout retention ratio",
 * default 1.0 = no dropout).  With keep_prob < 1 each probability p_ij is
 * kept with probability keep_prob and scaled by 1 / keep_prob, or zeroed;
 * LSE stays that of the probabilities before dropout.  The keep mask is a
 * function of (seed, offset, b, h, i, j) only, so the backward regenerates
 * it exactly: element (b, h, i, j) is kept iff u < round(keep_prob * 65536)
 * for u the 16-bit field j mod 8 (word (j mod 8) / 2, bits 16 * (j mod 2))
 * of Philox-4x32-10 (Salmon et al., SC'11) with key (seed mod 2^32,
 * seed / 2^32) and counter (c0, c1) = offset + j / 8 (mod 2^64), c2 = i,
 * c3 = (b*N + h) mod 2^32.  That is block offset + j / 8 of the Philox
 * stream with this seed and subsequence (b*N + h) * 2^32 + i, the
 * convention of torch's Philox engine: `offset` counts 128-bit blocks, and a
 * call reads blocks offset .. offset + ceil(Sk / 8) - 1 of each stream.
 * Pass the same (seed, offset) to fa_bwd; for a fresh mask advance `offset`
 * by at least ceil(Sk / 8), or change `seed`. */
typedef struct {
  uint64_t seed;
  uint64_t offset;
} fa_dropout;

typedef struct {
  int B, N, Sq, Sk, D;          /* batch, heads (head_num), query and key
                                   lengths, head dim                         */
  fa_layout layout;
  fa_dtype dtype;
} fa_shape;

/* Forward.  Writes out (layout/dtype of q) and lse (fp32 [B][N][Sq], natural
 * log, -inf for rows with no visible key).
 *   pse, mask : may be NULL (no bias / no mask).
 *   scale     : multiplies Q K^T (the 1/sqrt(d_k) of the guide's table; no
 *               default is assumed).
 *   keep_prob : retention probability in (0, 1]; 1 = no dropout.
 *   dropout   : the mask's generator key (see fa_dropout); required when
 *               keep_prob < 1, ignored (may be NULL) when keep_prob == 1.
 * Errors: FA_ERR_INVALID_ARG for null tensors, non-positive sizes, a
 * modality mask with Sq != Sk, a missing mask pointer, keep_prob outside
 * (0, 1] or a missing fa_dropout with keep_prob < 1; FA_ERR_UNSUPPORTED for
 * a bf16 / fp16 head dim other than 64 / 128. */
fa_status fa_fwd(const fa_shape* shape, const void* q, const void* k,
                 const void* v, const fa_pse* pse, const fa_mask* mask,
                 float scale, float keep_prob, const fa_dropout* dropout,
                 void* out, float* lse, void* stream);

/* Bytes of device workspace fa_bwd needs for this shape (fp32 dQ
 * accumulator plus per-row fp32 statistics).  0 on invalid shapes. */
size_t fa_bwd_workspace_size(const fa_shape* shape);

/* Backward: gradients of sum(dout * out) with respect to q, k and v, given
 * the forward's out and lse.  workspace must hold fa_bwd_workspace_size()
 * bytes (16-byte aligned); its contents on entry do not matter.  dq, dk, dv
 * are fully overwritten.  No gradient is produced for pse or the mask.
 * keep_prob and dropout must be those of the forward that produced out.
 * Errors as fa_fwd, plus FA_ERR_INVALID_ARG for a short workspace. */
fa_status fa_bwd(const fa_shape* shape, const void* q, const void* k,
                 const void* v, const void* out, const void* dout,
                 const float* lse, const fa_pse* pse, const fa_mask* mask,
                 float scale, float keep_prob, const fa_dropout* dropout,
                 void* dq, void* dk, void* dv, void* workspace,
                 size_t workspace_bytes, void* stream);

/* Backward without a caller-provided workspace (no counterpart on the source
 * pages; an addition of this library).  Some callers cannot call cudaMalloc:
 * code inside a host framework whose memory pool already holds the device
 * memory, or latency-critical loops that cannot afford the implicit
 * synchronisation of cudaMalloc / cudaFree.  This entry point allocates
 * nothing: its scratch (the fp32 dQ accumulator and per-row statistics that
 * fa_bwd keeps in its workspace) is a fixed device array of
 * FA_NOALLOC_SCRATCH_BYTES inside the library, reserved on every GPU that
 * loads the library until the process exits.
 *   - Arguments, results and errors are those of fa_bwd, except that a
 *     shape whose fa_bwd_workspace_size() exceeds FA_NOALLOC_SCRATCH_BYTES
 *     returns FA_ERR_UNSUPPORTED without launching anything.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process, so cudaDeviceReset
 *     is not supported while the library is in use.
 *   - Shapes with no (query, key) pair (B, N, Sq or Sk equal to 0) go to
 *     fa_bwd directly and never touch the array.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race on it and give wrong gradients.
 *     Calls on one stream, or otherwise ordered, are safe; the array keeps
 *     the previous call's contents and the backward clears what must start
 *     at zero. */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
fa_status fa_bwd_noalloc(const fa_shape* shape, const void* q, const void* k,
                         const void* v, const void* out, const void* dout,
                         const float* lse, const fa_pse* pse,
                         const fa_mask* mask, float scale, float keep_prob,
                         const fa_dropout* dropout, void* dq, void* dk,
                         void* dv, void* stream);

/* Bytes of the tile map for FA_MASK_BOOL with this shape and mask strides:
 * one byte per (b, h or 1 when mask_stride_h == 0, query tile, key tile). */
size_t fa_mask_tile_map_size(const fa_shape* shape, const fa_mask* mask);

/* Classifies every FA_TILE_M x FA_TILE_N tile of the bool mask as
 * 0 = no visible key, 1 = partly visible, 2 = fully visible, into
 * tile_map (fa_mask_tile_map_size bytes, device).  Reads the mask once. */
fa_status fa_build_mask_tile_map(const fa_shape* shape, const fa_mask* mask,
                                 uint8_t* tile_map, void* stream);

/* Builds the explicit cross-modal bool mask [B][S][S] (u8, 1 = may attend)
 * from modality_ids [B][S] with the 2x2 allow table and diagonal rule of
 * FA_MASK_MODALITY (the multimodal page's create_cross_modal_mask,
 * generalised).  Use with mask_stride_b = S*S, mask_stride_h = 0,
 * mask_stride_q = S. */
fa_status fa_build_modality_mask(int B, int S, const int32_t* modality_ids,
                                 const uint8_t allow[2][2], int allow_diag,
                                 uint8_t* mask_out, void* stream);

/* Synchronises `stream`, then returns and clears the device status word:
 * FA_ERR_TIMEOUT if a kernel gave up a bounded wait since the last call,
 * FA_ERR_CONCURRENT if a forward found its work counter shared with
 * another call (only possible with more than 64 forwards running at once),
 * FA_ERR_CUDA if the stream reported an error, else FA_OK. */
fa_status fa_sync_status(void* stream);

/* Static, human-readable name of a status code. */
const char* fa_status_string(fa_status status);

/* Library version string, e.g. "fa_b200 1.0 sm_100a". */
const char* fa_version(void);

/* Text of the last CUDA error behind an FA_ERR_CUDA returned to the calling
 * thread ("no error" if none).  Static storage; diagnostics only. */
const char* fa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
