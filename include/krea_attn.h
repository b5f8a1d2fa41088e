/*
 * krea_attn.h -- C ABI of the Krea 2 bidirectional attention core for B200 (sm_100a).
 *
 * One call computes, for every query token t of a [text, image] sequence and every
 * query head h,
 *
 *     out[b,t,h,:] = sigmoid(gate[b,t,h,:]) * sum_{j in A(t)} softmax_j(scale * s(t,j)) * v[b,j,h/rep,:]
 *
 * - bidirectional, non-causal attention with one running softmax state per row
 *   ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What it actually patches");
 * - grouped-query attention resolved inside the kernel: q head h reads kv head
 *   h / (Hq / Hkv), the repeat_interleave order (same section);
 * - three modes (krea_mode_t): dense; TileMix, where each 128x128 score tile is
 *   computed in FP16 or from INT8 codes by a static map (same page, sections
 *   "What it actually patches" and "The inputs that matter"); and scanline, a
 *   block-sparse mask in which text is global and an image token sees image tokens
 *   within window/2 latent rows ("Krea 2 Scanline Attention", section "What the
 *   mask actually is");
 * - the sigmoid(gate) multiply of the surrounding block fused into the epilogue;
 * - query slicing against full K/V ("LayerStream: Krea2 Chunking", section "What the
 *   node does to the block"): every slice of a 128-aligned query range gives the
 *   bit-identical rows of the single-slice call.
 *
 * Conventions shared by every entry point:
 * - Tensors are [batch, token, head, head_dim] with head_dim contiguous; the
 *   (batch, token, head) strides are given in ELEMENTS in krea_attn_params_t.
 *   q/k/v/gate/out must start on a 16-byte boundary and every stride times the
 *   element size must be a multiple of 16 bytes.
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   never frees or keeps them. The only memory the library owns is its tile-map
 *   cache (device copies of the block-sparse lists; at most 8 entries per device,
 *   released by krea_attn_clear_cache()).
 * - Work is enqueued on `stream` and runs asynchronously; the only blocking step
 *   is a host-to-device copy when a tile map is built for the first time.
 * - Every call returns KREA_OK (0) or a negative krea_status_t; no C++ exception
 *   crosses the ABI. krea_attn_error_string() names a code. Errors detected on
 *   the device (a bounded wait that ran out) are written to params->status.
 */
#ifndef KREA_ATTN_H_
#define KREA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KREA_API __attribute__((visibility("default")))
#else
#define KREA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define KREA_ATTN_ABI_VERSION 3
#define KREA_ATTN_TILE 128

typedef enum {
  KREA_MODE_DENSE = 0,     /* every key for every query */
  KREA_MODE_TILEMIX = 1,   /* per-tile FP16 / INT8 routing by a static map */
  KREA_MODE_SCANLINE = 2   /* block-sparse scanline mask over 128-token tiles */
} krea_mode_t;

typedef enum { KREA_F16 = 0, KREA_BF16 = 1, KREA_F32 = 2 } krea_dtype_t;

/* TileMix patterns ("Krea 2 TileMix Attention", section "The inputs that matter"):
 * zero keeps every tile FP16; band sends a `percentage` share of the left-over
 * image-image tiles (off the diagonal band) to INT8, farthest from the diagonal
 * first; one sends all of them to INT8. */
typedef enum { KREA_PATTERN_ZERO = 0, KREA_PATTERN_BAND = 1, KREA_PATTERN_ONE = 2 } krea_pattern_t;

typedef enum {
  KREA_OK = 0,
  KREA_ERR_INVALID_ARG = -1,     /* bad shape, stride, alignment, window, slice or percentage */
  KREA_ERR_UNSUPPORTED = -2,     /* fp32 inputs, head_dim not 64/128, Hq % Hkv != 0, INT8 with head_dim 64 */
  KREA_ERR_WORKSPACE = -3,       /* workspace missing or smaller than krea_attn_workspace_bytes() */
  KREA_ERR_CUDA = -4,            /* a CUDA runtime call or a launch failed */
  KREA_ERR_DEVICE_TIMEOUT = -5,  /* written to *status: a bounded wait in a kernel ran out */
  KREA_ERR_DEVICE_BOUNDS = -6,   /* written to *status: a kernel met an out-of-range index */
  KREA_ERR_NO_DEVICE = -7,       /* no CUDA device, or not an sm_100 device */
  KREA_ERR_TOO_LARGE = -8        /* a fixed limit of the call: krea_attn_fwd_noalloc's scratch, the exchange's size */
} krea_status_t;

/* Kind bits of one tile of a map (krea_attn_get_map). */
#define KREA_KIND_MASKED 1  /* some key slot of the tile is padding or not admitted */
#define KREA_KIND_INT8 2    /* the tile's scores come from INT8 codes */

typedef struct {
  int32_t abi_version;   /* must be KREA_ATTN_ABI_VERSION */
  int32_t batch;         /* B >= 1 */
  int32_t num_q_heads;   /* Hq >= 1 */
  int32_t num_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;      /* 64 or 128 (INT8 tiles need 128) */
  int32_t q_start;       /* first query token of this slice, a multiple of 128 */
  int32_t q_len;         /* query tokens in this slice; 0 means up to the end */
  int32_t in_dtype;      /* krea_dtype_t of q, k, v, gate: KREA_F16 or KREA_BF16 */
  int32_t out_dtype;     /* KREA_F32 or the input dtype */
  int64_t q_stride[3];   /* (batch, token, head) strides of q, in elements */
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t gate_stride[3];
  int64_t out_stride[3];
  float softmax_scale;   /* 0 -> 1/sqrt(head_dim) */
  /* TileMix */
  int32_t pattern;       /* krea_pattern_t */
  float percentage;      /* share of left-over image-image tiles sent to INT8, in [0, 1] */
  int32_t band_blocks;   /* key blocks on each side of the diagonal kept FP16; < 0 -> 2 */
  int32_t smooth_k;      /* centre K per (batch, kv head, channel) before quantising */
  int32_t qk_fp32_accumulate; /* accepted and recorded: QK^T always accumulates in fp32 */
  /* scanline */
  int32_t window;        /* odd, 1..255: image tokens see image rows within window/2 */
  int32_t tile_aligned;  /* 1: every valid pair inside an active tile is admitted */
  int32_t text_pad;      /* text slot size, multiple of 128, >= text_len; 0 -> max(512, ceil128(T)) */
  /* scratch and status */
  void* workspace;       /* device memory, krea_attn_workspace_bytes() bytes; TileMix only */
  size_t workspace_bytes;
  int32_t* status;       /* optional device int32, zero before the call: a kernel that gives up writes a
                            negative code; a kernel that finds it nonzero does no work */
  int64_t debug_wait_limit; /* SM clock cycles a kernel waits on one barrier before giving up; 0 -> 2e9 */
  int32_t debug_flags;   /* bit 0: one softmax warp waits on a barrier nothing arrives at (tests the bounded wait);
                            bit 1: every exponential through the FMA-pipe polynomial (tests its accuracy) */
  float* lse;            /* optional device fp32 [B, Hq, L], 4-byte aligned: for every valid query row of the
                            slice, ln sum_j exp(softmax_scale * s_ij) over its admitted keys (the softmax
                            normaliser a backward pass needs); rows outside the slice are not written */
  int32_t overlap_previous; /* 1: the attention kernel of this call may start while the work enqueued before
                            it on the stream still runs (CUDA programmatic dependent launch), so its CTAs fill
                            the SMs the previous kernel's last wave leaves idle. The caller guarantees that
                            the earlier work writes nothing this call reads and touches none of the rows this
                            call writes: e.g. the next query slice of the same attention ("Krea 2 TileMix
                            Attention (FP16/INT8 tiles)": the queries are processed in slices). The call
                            still completes after the earlier work (every CTA waits for it before it
                            exits), so later work on the stream sees both. Ignored for TileMix, whose
                            quantiser runs first in the same call. 0: ordinary stream order. */
} krea_attn_params_t;

/* Fill `p` with the defaults for a contiguous [B, L, H, d] layout. */
KREA_API void krea_attn_default_params(krea_attn_params_t* p, int batch, int num_q_heads, int num_kv_heads,
                              int head_dim, int text_len, int grid_h, int grid_w);

/* The attention forward. q [B,L,Hq,d], k and v [B,L,Hkv,d], gate [B,L,Hq,d] or NULL,
 * out [B,L,Hq,d] (only rows q_start .. q_start+q_len-1 are written); L = text_len +
 * grid_h * grid_w, text tokens first, image tokens row-major on a grid_h x grid_w grid.
 * mode is a krea_mode_t. TileMix needs params->workspace. */
KREA_API int krea_attn_fwd(const void* q, const void* k, const void* v, const void* gate, void* out,
                  int text_len, int grid_h, int grid_w, int mode, const krea_attn_params_t* params,
                  void* stream);

/* Bytes of caller-allocated workspace krea_attn_fwd needs (0 if none): only TileMix
 * calls need any, for the smooth_k centred keys ("Krea 2 TileMix Attention (FP16/INT8
 * tiles)", section "The inputs that matter") and the INT8 codes and block scales of
 * the tiles the map sends to INT8 (section "What it actually patches"; the
 * per-(batch, head, 128-token block) absmax/127 scheme is this library's, the pages
 * give none). Returns 0 for other modes or invalid params; pure host arithmetic. */
KREA_API size_t krea_attn_workspace_bytes(int text_len, int grid_h, int grid_w, int mode,
                                 const krea_attn_params_t* params);

/* Byte offsets inside the workspace (TileMix) of:
 *   kc  centred keys k - mean, [B, L, Hkv, d], input dtype (smooth_k only)
 *   q8  INT8 query codes [B, L, Hq, d];  k8 INT8 key codes [B, L, Hkv, d]
 *   sq  query scales [B, Hq, nt] f32;    sk key scales [B, Hkv, nt] f32 (nt = ceil(L/128))
 *   mu  key mean [B, Hkv, d] f32;        part  per-chunk partial sums (f64) */
typedef struct {
  size_t kc, q8, k8, sq, sk, mu, part, total;
} krea_attn_ws_layout_t;
KREA_API int krea_attn_workspace_layout(int text_len, int grid_h, int grid_w, int mode,
                               const krea_attn_params_t* params, krea_attn_ws_layout_t* out);

/* Size of the tile map: *n_tiles query tiles (the logical sequence, text slot
 * included for scanline) and *nnz listed (query tile, key tile) pairs. The map is
 * the 128-tile block map of "Krea 2 Scanline Attention", section "What the mask
 * actually is" (scanline), or the per-tile FP16/INT8 routing of "Krea 2 TileMix
 * Attention (FP16/INT8 tiles)", sections "What it actually patches" and "The inputs
 * that matter" (TileMix); dense lists every pair. Host work; needs no GPU;
 * KREA_ERR_INVALID_ARG for a bad geometry or params. */
KREA_API int krea_attn_map_size(int text_len, int grid_h, int grid_w, int mode, const krea_attn_params_t* params,
                       int32_t* n_tiles, int32_t* nnz);

/* Copy the tile map into HOST buffers: row_ptr[n_tiles + 1], col[nnz] (key tiles,
 * ascending per row) and kind[nnz] (KREA_KIND_* bits). `capacity` is the length of
 * col and kind (KREA_ERR_INVALID_ARG when smaller than nnz, or a NULL buffer). The
 * map rules are those of krea_attn_map_size: the scanline block map ("Krea 2
 * Scanline Attention", section "What the mask actually is") or TileMix's per-tile
 * routing ("Krea 2 TileMix Attention (FP16/INT8 tiles)", sections "What it actually
 * patches" and "The inputs that matter"). The caller owns the buffers; pure host
 * work, needs no GPU. */
KREA_API int krea_attn_get_map(int text_len, int grid_h, int grid_w, int mode, const krea_attn_params_t* params,
                      int32_t* row_ptr, int32_t* col, uint8_t* kind, int32_t capacity);

/* Build the same tile map on the DEVICE, asynchronously on `stream`, into device
 * buffers row_ptr[n_tiles + 1], col[capacity] and kind[capacity], laid out as
 * krea_attn_get_map's (map rules: "Krea 2 Scanline Attention", section "What the
 * mask actually is"; "Krea 2 TileMix Attention (FP16/INT8 tiles)", sections "What
 * it actually patches" and "The inputs that matter"). n_tiles comes from
 * krea_attn_map_size, and capacity = n_tiles * n_tiles always suffices. row_ptr is
 * always written (row_ptr[n_tiles] = nnz); when nnz > capacity, col and kind are
 * left untouched and params->status, if set, receives KREA_ERR_DEVICE_BOUNDS.
 * No host work beyond validation, no allocation, no copy. */
KREA_API int krea_attn_build_map_device(int text_len, int grid_h, int grid_w, int mode,
                                        const krea_attn_params_t* params, int32_t* row_ptr, int32_t* col,
                                        uint8_t* kind, int32_t capacity, void* stream);

/* QK prologue: RMSNorm, then the 3-axis rotary embedding -- the two steps the
 * pages keep stock on q and k right before the attention core ("Krea 2 TileMix
 * Attention (FP16/INT8 tiles)", section "What it actually patches"; the pages give
 * no formula: the readings below are this library's), in one pass over HBM:
 *   y = rope(x * gamma / sqrt(mean(x^2) + eps))   per (batch, token, head) vector.
 * rope turns adjacent channel pairs (2i, 2i+1) of three consecutive channel
 * groups of axes_dim[0], axes_dim[1], axes_dim[2] channels (text index, image row,
 * image column; the channels after them pass unchanged) by
 * pos[t][a] * theta^(-2i / axes_dim[a]) radians. */
typedef struct {
  int32_t axes_dim[3]; /* even; sum <= head_dim and a multiple of 4 */
  float theta;         /* > 0 */
  float eps;           /* >= 0, added to the mean square */
} krea_rope_params_t;

/* (head_dim/4, 3 head_dim/8, 3 head_dim/8) channels, theta 10000, eps 1e-6. */
KREA_API void krea_attn_default_rope(krea_rope_params_t* rope, int head_dim);

/* Rotary positions of the joint [text, image] sequence, the layout this library
 * takes for the 3-axis RoPE the pages name ("Krea 2 TileMix Attention (FP16/INT8
 * tiles)", section "What it actually patches": QK RMSNorm and 3-axis RoPE run right
 * before the core; the pages give no layout): text token t at (t, 0, 0), image token
 * at grid row r, column c at (0, r, c), image tokens row-major after the text.
 * Writes pos[L][3] int32 (L = text_len + grid_h * grid_w) into a HOST buffer of
 * `capacity` rows; KREA_ERR_INVALID_ARG for a bad geometry, a NULL pointer or
 * capacity < L. Pure host work; needs no GPU. Other layouts are passed to
 * krea_attn_rope_table directly. */
KREA_API int krea_attn_rope_positions(int text_len, int grid_h, int grid_w, int32_t* pos, int32_t capacity);

/* Rotary table of a geometry: table[t][j] = (cos, sin) of pair j's angle for
 * token t (pairs numbered axis by axis), from pos [tokens][3] int32 (device),
 * angles and trigonometry in fp64, stored as fp32 in table
 * [tokens][n_pairs][2] (device, 16-byte aligned, n_pairs = sum(axes_dim) / 2).
 * Build it once per geometry: every block and both q and k reuse it. */
KREA_API int krea_attn_rope_table(const int32_t* pos, int tokens, const krea_rope_params_t* rope, float* table,
                                  void* stream);

/* y = rope(rmsnorm(x)) on device tensors x, y [batch, tokens, heads, head_dim]
 * (element strides x_stride / y_stride over (batch, token, head), head_dim
 * contiguous, rows 16-byte aligned; y may be x: in place). dtype KREA_F16 or
 * KREA_BF16 for both; computed in fp32, rounded once. gamma: head_dim fp32
 * weights (device) or NULL for ones. table: from krea_attn_rope_table with the
 * same rope params. head_dim 64 or 128.
 * If codes is not NULL, the pass also writes the TileMix INT8 codes of the stored
 * y, codes [batch, tokens, heads, head_dim] contiguous, and scales [batch, heads,
 * ceil(tokens / 128)] (one per 128-token block: absmax / 127), decided exactly as
 * krea_attn_quantize decides them for queries. */
KREA_API int krea_attn_qk_prologue(const void* x, void* y, const float* gamma, const float* table, int batch,
                                   int tokens, int heads, int head_dim, int dtype, const int64_t* x_stride,
                                   const int64_t* y_stride, const krea_rope_params_t* rope, int8_t* codes,
                                   float* scales, void* stream);

/* The attention forward on RAW query projections, with the query half of the QK
 * prologue fused into the core: each CTA normalises and rotates its Q tile in
 * shared memory right before the first QK^T, so q makes no extra HBM round trip
 * ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section "What it actually
 * patches": QK RMSNorm and the 3-axis RoPE run on q and k right before the core).
 * The result equals krea_attn_qk_prologue(q_raw) followed by krea_attn_fwd bit for
 * bit: the fused step repeats the prologue pass's arithmetic in the same order.
 *   q_raw   [B, L, Hq, d] raw projections (layout and strides as q of krea_attn_fwd)
 *   q_gamma d fp32 RMSNorm weights (device, 4-byte aligned) or NULL for ones
 *   table   the rotary table of this geometry from krea_attn_rope_table (device,
 *           16-byte aligned, row t = token t of the sequence), built with `rope`
 *   rope    axes_dim, theta (the table's) and eps (RMSNorm)
 *   k       keys ALREADY through the prologue (krea_attn_qk_prologue on k: each
 *           kv head's rows are read by every query tile, so they are rotated once)
 *   v, gate, out, text_len, grid_h, grid_w, params, stream: as krea_attn_fwd.
 * Modes KREA_MODE_DENSE and KREA_MODE_SCANLINE; TileMix returns
 * KREA_ERR_UNSUPPORTED (its INT8 query codes are decided on the stored prologue
 * output: use krea_attn_qk_prologue with codes, then krea_attn_fwd). Other errors as
 * krea_attn_fwd, and KREA_ERR_INVALID_ARG for a NULL or misaligned table, a
 * misaligned gamma or invalid rope params. The caller owns every buffer; nothing
 * is kept after the call. */
KREA_API int krea_attn_fwd_rope_q(const void* q_raw, const float* q_gamma, const float* table,
                                  const krea_rope_params_t* rope, const void* k, const void* v, const void* gate,
                                  void* out, int text_len, int grid_h, int grid_w, int mode,
                                  const krea_attn_params_t* params, void* stream);

/* ---- sequence <-> head exchange (sequence-parallel callers) ----------------
 * A caller whose block holds the joint [text, image] sequence split by token
 * across `world` ranks (rank r: tokens [r * tokens_per_rank, (r + 1) *
 * tokens_per_rank)) turns it into a split by head before the attention core and
 * back after it. Every head of the core is independent, and query head h reads
 * kv head h / (Hq / Hkv) ("Krea 2 TileMix Attention (FP16/INT8 tiles)", section
 * "What it actually patches": the key/value heads are repeated to the query
 * heads), so rank j can run the ordinary call on query heads [j Hq / world,
 * (j + 1) Hq / world) and kv heads [j Hkv / world, (j + 1) Hkv / world) over the
 * whole sequence. The pages describe no multi-GPU split; this is the plain one.
 *
 * The exchange is a push: each rank stores its rows straight into the
 * destination buffers of every rank (peer memory over NVLink, or this device's
 * own memory), with no packing pass and no library collective. The caller
 * orders the ranks around it: no rank may read a destination before every rank's
 * exchange into it has completed (a stream-ordered barrier, e.g. a one-element
 * all-reduce), and no rank may overwrite a destination that its owner still
 * reads. The stores are performed when the launch completes on `stream`.
 *
 * Ownership: the caller owns the source, every destination and the stream; the
 * library keeps no pointer after the call returns. Source and destinations must
 * not overlap. Errors, returned before anything is launched or written:
 * KREA_ERR_INVALID_ARG (world, rank, tokens_per_rank or reserved out of range,
 * a NULL or misaligned pointer, a stride that is not a positive multiple of 16
 * bytes, heads not divisible by world, an unknown dtype), KREA_ERR_UNSUPPORTED
 * (head_dim not 64 or 128; fp32 into the prologue), KREA_ERR_TOO_LARGE,
 * KREA_ERR_NO_DEVICE; KREA_ERR_CUDA if the launch fails. Destination sizes are
 * not checked: each dst[j] must hold the shape the rule below writes. */
#define KREA_EXCHANGE_MAX_RANKS 16
typedef struct {
  int32_t world;            /* ranks sharing the sequence, 1 .. KREA_EXCHANGE_MAX_RANKS */
  int32_t rank;             /* this rank, 0 .. world - 1 */
  int32_t tokens_per_rank;  /* tokens of every shard (> 0); the sequence holds world * tokens_per_rank */
  int32_t reserved;         /* 0 */
  void* dst[KREA_EXCHANGE_MAX_RANKS]; /* dst[j]: rank j's destination buffer as this process addresses it
                                         (device memory of this GPU or an opened IPC mapping of a peer's);
                                         16-byte aligned; entries past world are ignored */
  int64_t dst_stride[3];    /* element strides (b, token, head) shared by every dst[j]; multiples of 16 bytes */
} krea_exchange_t;

/* Token shard -> head shards. x: this rank's rows [batch, tokens_per_rank, heads,
 * head_dim] (device, strides x_stride over (b, token, head), head_dim contiguous).
 * heads % world == 0; row (b, t, h) is copied unchanged to dst[h / (heads /
 * world)] at (b, rank * tokens_per_rank + t, h mod (heads / world)). dtype
 * KREA_F16, KREA_BF16 or KREA_F32; head_dim 64 or 128. One batch entry of x
 * holds fewer than 2^35 bytes (KREA_ERR_TOO_LARGE otherwise). */
KREA_API int krea_attn_seq_to_heads(const void* x, int batch, int heads, int head_dim, int dtype,
                                    const int64_t* x_stride, const krea_exchange_t* ex, void* stream);

/* Head shard -> token shards, the inverse. y: this rank's heads over the whole
 * sequence [batch, world * tokens_per_rank, heads, head_dim]; row (b, t, h) goes
 * to dst[t / tokens_per_rank] at (b, t mod tokens_per_rank, rank * heads + h).
 * Same types and limits as krea_attn_seq_to_heads. */
KREA_API int krea_attn_heads_to_seq(const void* y, int batch, int heads, int head_dim, int dtype,
                                    const int64_t* y_stride, const krea_exchange_t* ex, void* stream);

/* The QK prologue of krea_attn_qk_prologue on this rank's token shard x [batch,
 * tokens_per_rank, heads, head_dim], its output stored as krea_attn_seq_to_heads
 * stores rows: y of row (b, t, h) lands in dst[h / (heads / world)] at (b, rank *
 * tokens_per_rank + t, h mod (heads / world)). The rotation of row t uses table
 * row rank * tokens_per_rank + t: the table covers the whole sequence. dtype
 * KREA_F16 or KREA_BF16; no INT8 codes in this form. */
KREA_API int krea_attn_qk_prologue_to_heads(const void* x, const float* gamma, const float* table, int batch,
                                            int heads, int head_dim, int dtype, const int64_t* x_stride,
                                            const krea_rope_params_t* rope, const krea_exchange_t* ex,
                                            void* stream);

/* Destination buffers other processes can map (CUDA IPC on one node).
 * krea_attn_ipc_alloc allocates `bytes` of device memory on the current device
 * (a dedicated allocation: the handle maps exactly this buffer) and writes its
 * handle (KREA_IPC_HANDLE_BYTES opaque bytes) to `handle`; krea_attn_ipc_free
 * releases it. krea_attn_ipc_open maps another process's handle into this one
 * (not one of this process's own allocations) and krea_attn_ipc_close unmaps
 * it. NULL arguments or zero bytes return KREA_ERR_INVALID_ARG, a missing sm_100
 * device KREA_ERR_NO_DEVICE; CUDA failures return KREA_ERR_CUDA with nothing
 * allocated or mapped. */
#define KREA_IPC_HANDLE_BYTES 64
KREA_API int krea_attn_ipc_alloc(size_t bytes, void** ptr, void* handle);
KREA_API int krea_attn_ipc_free(void* ptr);
KREA_API int krea_attn_ipc_open(const void* handle, void** ptr);
KREA_API int krea_attn_ipc_close(void* ptr);

/* Run only the TileMix quantiser into params->workspace (device memory of
 * krea_attn_workspace_bytes() bytes, 16-byte aligned, owned by the caller), laid out
 * as krea_attn_workspace_layout() says: the key mean per (batch, kv head, channel)
 * and the centred keys k - mean (smooth_k: "Krea 2 TileMix Attention (FP16/INT8
 * tiles)", section "The inputs that matter"), then the symmetric INT8 codes and
 * absmax/127 scales of q and of the (centred) keys per (batch, head, 128-token
 * block), the scheme this library fixes (the pages give none). q, k: device
 * tensors as for krea_attn_fwd; head_dim 128. Asynchronous on `stream`. Errors:
 * KREA_ERR_INVALID_ARG (pointers, strides, geometry), KREA_ERR_UNSUPPORTED
 * (head_dim), KREA_ERR_WORKSPACE, KREA_ERR_NO_DEVICE, KREA_ERR_CUDA. */
KREA_API int krea_attn_quantize(const void* q, const void* k, int text_len, int grid_h, int grid_w,
                       const krea_attn_params_t* params, void* stream);

/* The same attention as krea_attn_fwd, for callers that cannot allocate device
 * memory while they run (an arena or pool that forbids cudaMalloc/cudaFree, which
 * synchronise the device; a host framework that owns all device memory; a serving
 * loop that must not block on the allocator). It allocates, caches and frees
 * nothing and copies nothing from the host: the tile map is built on `stream` by
 * the device map builder (the same map krea_attn_fwd caches, bit for bit) and,
 * with the TileMix workspace, lives in one fixed 64 MiB array in device memory
 * declared by the library, held on every GPU that loads the library until the
 * process exits; params->workspace is ignored. Results equal krea_attn_fwd's bit
 * for bit. Shapes whose map (4 (n_tiles + 1) + 4 n_tiles^2 bytes) plus workspace
 * exceed 64 MiB return KREA_ERR_TOO_LARGE before any launch (a 48/12-head TileMix
 * call fits up to about 1 MP; dense and scanline calls fit far beyond 4 MP). All
 * calls share the array, so calls whose GPU work overlaps (two streams, or two
 * threads on one device) race and must not be issued; calls on one stream are
 * ordered (params->overlap_previous is ignored: the attention reads the map
 * built just before it). Each call rewrites everything it reads, nothing needs clearing. The
 * first call on a device looks up the array's device address; make it before any
 * CUDA stream capture on that device. The pages describe no counterpart of this
 * entry point. */
KREA_API int krea_attn_fwd_noalloc(const void* q, const void* k, const void* v, const void* gate, void* out,
                                   int text_len, int grid_h, int grid_w, int mode,
                                   const krea_attn_params_t* params, void* stream);

/* Backward of krea_attn_fwd for dense and scanline calls (TileMix INT8 codes
 * have no gradient): with P the softmax weights over the admitted keys (from the
 * forward's lse), O = P v and out = sigmoid(gate) O,
 *   dv = P^T dO, dq = scale dS k, dk = scale dS^T q, dgate = dout out (1 - sigmoid(gate)),
 *   dO = dout sigmoid(gate), dS = P (dO v^T - rowsum(dout out)),
 * dk and dv summed over the query heads of each kv head.
 * Inputs: q, k, v, gate as given to the forward (params strides and dtype), out
 * and dout contiguous [B, L, Hq, d] of params->out_dtype, lse [B, Hq, L] fp32 from
 * the forward (params->lse). Outputs, all fp32 and contiguous: dq [B, L, Hq, d]
 * (zeroed, then accumulated), dk and dv [B, L, Hkv, d], dgate [B, L, Hq, d] (may
 * be NULL; ignored without a gate). scratch: krea_attn_bwd_scratch_bytes() bytes
 * of device memory, 256-byte aligned. The whole sequence only (q_start 0, q_len 0
 * or L); head_dim 64 or 128. */
KREA_API size_t krea_attn_bwd_scratch_bytes(int text_len, int grid_h, int grid_w, const krea_attn_params_t* params);
KREA_API int krea_attn_bwd(const void* q, const void* k, const void* v, const void* gate, const void* out,
                           const void* dout, const float* lse, float* dq, float* dk, float* dv, float* dgate,
                           void* scratch, int text_len, int grid_h, int grid_w, int mode,
                           const krea_attn_params_t* params, void* stream);

/* Release every cached tile map on every device. */
KREA_API void krea_attn_clear_cache(void);

/* Static text for a krea_status_t (never NULL; "unknown error" for other codes).
 * The codes replace the pages' silent dense fallbacks ("Krea 2 TileMix Attention
 * (FP16/INT8 tiles)", section "Where people get burned"): an unsupported input is
 * an error, never a different computation. */
KREA_API const char* krea_attn_error_string(int code);

/* KREA_ATTN_ABI_VERSION of the loaded library. */
KREA_API int krea_attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KREA_ATTN_H_ */
