/*
 * lcsa.h - C ABI of the B200 (sm_100a) locality-constrained block-sparse
 * causal attention (LCSA) hot path of FlashVSR's one-step streaming DiT.
 *
 * Sources of the operations (page title, section):
 *  - "FlashVSR 是怎么工作的" (vsr-hover-compare learn.html), 2.2 LCSA:
 *    WindowPartition3D into (2,8,8) blocks, local block mask (default
 *    local_range 11), block mean pooling, draft scores q.k/sqrt(D), -inf
 *    outside the mask, top-k, block_sparse_attn_func over the kept pairs.
 *  - same page, 2.3 streaming + KV cache: keep the newest kv_len block-layers,
 *    drop the oldest one per step.
 *  - reading notes "FlashVSR: Towards Real-time Diffusion-Based Streaming
 *    Video Super Resolution", 关键设计 1 (causal mask), 2 (block-sparse
 *    attention on top-k 128x128 block pairs), 3 (local window, the
 *    Boundary-Preserved and Boundary-Truncated rules).
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers on the current CUDA device,
 *    allocated and owned by the caller; the library never allocates or frees
 *    device memory.  Tensor pointers must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *    NULL = legacy default stream).
 *  - Return value: LCSA_OK, or an LCSA_ERR_* code for a synchronous argument
 *    or launch error; nothing is enqueued when an error is returned.
 *  - Device-side errors (a watchdog that expired, an out-of-range kept index)
 *    are OR-ed into *d_status (a device int32 the caller zeroes and reads
 *    after synchronising); d_status may be NULL to ignore them.
 *  - Token layout of q/k/v/out: bf16 [heads][frames][8*grid_h][8*grid_w][128],
 *    frames = 2 per block-layer.  Block b of a layer is (by, bx) =
 *    (b / grid_w, b % grid_w); token n of a block is
 *    (t, y, x) = (n / 64, (n / 8) % 8, n % 8) (row-major in (t, y, x)).
 *  - Key-block indices are LOGICAL: j = layer * grid_h*grid_w + b, layer 0
 *    being the oldest resident layer of the cache.
 *  - Only compute capability 10.0 (B200) is supported.
 */
#ifndef LCSA_H
#define LCSA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum lcsa_status {
    LCSA_OK = 0,
    LCSA_ERR_INVALID_ARG = 1,
    LCSA_ERR_UNSUPPORTED_DEVICE = 2,
    LCSA_ERR_CUDA = 3,
    /* device status bits (OR-ed into *d_status) */
    LCSA_ERR_TIMEOUT = 4,    /* a bounded wait inside a kernel gave up */
    LCSA_ERR_BAD_INDEX = 8   /* a kept index / count was out of range */
};

/* lcsa_params.flags */
#define LCSA_FLAG_FORCE_TIMEOUT 1 /* test hook: the first consumer wait of
                                     lcsa_attention (lcsa_params.flags) or of
                                     every CTA of lcsa_cache_append (its flags
                                     argument) gives up at once */
#define LCSA_FLAG_PDL 2           /* launch as a programmatic dependent of the
                                     kernel that precedes the call in the stream,
                                     so that it starts while that kernel finishes.
                                     lcsa_draft_mask reads q_tok, writes
                                     scores_opt / qmean_opt / q_rot_opt and
                                     reads the key
                                     means of the layers older than the newest
                                     max(q_layers, cache->appended) before
                                     waiting for that kernel
                                     (griddepcontrol.wait), and reads the other
                                     key means and writes the kept lists only
                                     after; lcsa_attention reads and writes
                                     nothing before the wait.  Set the flag only
                                     when the preceding kernel neither writes
                                     q_tok or those older key means nor touches
                                     scores_opt / qmean_opt / q_rot_opt, e.g.
                                     when it is the
                                     cache append of the same chunk (before the
                                     draft: it writes only the cache->appended
                                     newest layers) or the draft (before the
                                     attention).  lcsa_cache_append
                                     (flags argument) writes the ring before the
                                     wait and waits only at its end: set it only
                                     when the preceding kernel writes neither
                                     k_tok nor v_tok and the new layers fit the
                                     ring's spare slots
                                     (n_layers <= capacity - window), e.g. when it
                                     is the previous chunk's lcsa_attention. */

#define LCSA_HEAD_DIM 128
#define LCSA_BLOCK_TOKENS 128
#define LCSA_MAX_CANDIDATES 4096 /* allowed key blocks per query block */
#define LCSA_MAX_SEGMENTS 256    /* segments of one lcsa_segment_mask call */

/* Rotary position embedding of q and k (see lcsa_params.rope and the rope
 * argument of lcsa_cache_append).  Named by the reading notes (背景, 关键设计
 * 3) without a layout; the layout taken: each adjacent pair of dimensions
 * (2i, 2i+1) of the 128-dim head turns by pos * w_i, the 64 pairs split into
 * three axis bands: pairs [0, 22) over the latent frame's position in the
 * stream (frame0 + the frame index inside the call's tensor), [22, 43) over the
 * token row, [43, 64) over the token column; inside a band of n pairs
 * w_i = base^(-i/n).  cos and sin are evaluated in fp64 and rounded to fp32,
 * the rotation is computed in fp32 (each product and sum rounded once) and
 * rounded to bf16: the rotated q and k are the bf16 values every later step
 * (block means, scores, attention, the ring) uses. */
typedef struct lcsa_rope {
    float base;      /* e.g. 10000 (> 1); 0 disables the rotation */
    int32_t frame0;  /* stream position of the first latent frame of the call's tokens, >= 0;
                        every position (frame0 + frames of the call, token rows and
                        columns) must stay <= 2^20, else LCSA_ERR_INVALID_ARG */
} lcsa_rope;

typedef struct lcsa_params {
    int32_t heads;       /* H >= 1 */
    int32_t head_dim;    /* must be 128 */
    int32_t grid_h;      /* blocks per latent frame along y (tokens / 8) */
    int32_t grid_w;      /* blocks per latent frame along x (tokens / 8) */
    int32_t q_layers;    /* query block-layers: the newest q_layers of the cache */
    int32_t local_range; /* window side in blocks (odd, e.g. 11); <= 0: no window */
    int32_t local_mode;  /* 0 Boundary-Preserved (window shifted inside the
                            grid), 1 Boundary-Truncated (|i-j| <= range/2) */
    int32_t topk;        /* kept key blocks per query block, >= 1; also the
                            row stride of kept_idx */
    float scale;         /* softmax scale; 0 -> 1/sqrt(head_dim) */
    int32_t flags;       /* LCSA_FLAG_*; 0 in normal use */
    lcsa_rope rope;      /* rotation of q (draft and attention); base 0: none.
                            frame0: stream position of q_tok's first frame */
} lcsa_params;

/* Ring of block-layers, caller-owned device buffers:
 *   k, v   bf16 [capacity][heads][grid_h*grid_w][128 tokens][128]
 *   kmean  fp32 [capacity][heads][grid_h*grid_w][128]  (block means of k)
 * Slot of logical layer L: (oldest + L) % capacity.  `oldest` and `count`
 * are host-side state updated by lcsa_cache_append; start from 0, 0.
 * At most `window` layers are resident (kv_len + layers of one step); the
 * slots beyond the window (capacity - window of them) are spares: a new layer
 * goes into the slot after the newest one, so that it never overwrites a layer
 * of the previous window (what lets an append overlap the previous step, see
 * LCSA_FLAG_PDL). window = 0 means window = capacity (no spare slot). */
typedef struct lcsa_kv_cache {
    void *k;
    void *v;
    float *kmean;
    int32_t capacity; /* slots: window, plus spares */
    int32_t oldest;
    int32_t count;    /* resident layers, <= window */
    int32_t heads;
    int32_t grid_h;
    int32_t grid_w;
    int32_t window;   /* 0 < window <= capacity, or 0 for capacity */
    int32_t appended; /* layers written by the last lcsa_cache_append (set by
                         it; start from 0): a draft chained after that append
                         (LCSA_FLAG_PDL) reads them only after waiting for it */
} lcsa_kv_cache;

/*
 * lcsa_cache_append - append n_layers block-layers of keys and values
 * (learn.html 2.3: the cache keeps the newest layers and drops the oldest).
 *   k_tok, v_tok: bf16 token layout [heads][2*n_layers][8*grid_h][8*grid_w][128].
 * Each layer is written in block layout (partition of learn.html 2.2) into
 * the slot after the newest layer, together with its fp32 block means of k;
 * when `window` layers are resident the oldest is dropped and `oldest`
 * advances (without spare slots its slot is the one reused).
 *   flags: 0, LCSA_FLAG_PDL and/or LCSA_FLAG_FORCE_TIMEOUT (see there).
 *   d_status: device word (may be NULL); LCSA_ERR_TIMEOUT is OR-ed into it
 *   when a bounded wait for a copy gave up.
 *   rope: NULL or base 0 for none; else k is rotated (lcsa_rope) before it is
 *   stored and averaged, frame0 being the stream position of k_tok's first
 *   frame.
 * The copies are TMA loads of whole blocks and bulk stores into the ring.
 * Updates cache->oldest/count/appended on the host when the copy is enqueued,
 * so calls on one cache must be serialised by the caller.
 * 1 <= n_layers <= window.
 */
int lcsa_cache_append(lcsa_kv_cache *cache, const void *k_tok, const void *v_tok,
                      int32_t n_layers, int32_t flags, const lcsa_rope *rope, int32_t *d_status,
                      void *stream);

/*
 * lcsa_draft_mask - the draft mask of learn.html 2.2, one row per
 * (head, query block).  Query block i of layer ql sits at key layer
 * count - q_layers + ql.  Steps: fp32 block mean of q (fixed-order sum,
 * times 1/128); for every key block j allowed by the local window (same
 * spatial window on every layer, rule per local_mode) and by block causality
 * (key layer <= query layer): s = mean_q . kmean_j * scale, in fp32; keep the
 * min(topk, allowed) largest s, ties to the lower j.  With p->rope, q is
 * rotated (lcsa_rope) before its block means.
 *   q_tok      bf16 token layout [heads][2*q_layers][8*grid_h][8*grid_w][128]
 *   kept_idx   int32 [heads][q_layers*grid_h*grid_w][topk]: kept j ascending,
 *              padded with -1
 *   kept_cnt   int32 [heads][q_layers*grid_h*grid_w]
 *   scores_opt fp32 [heads][Nq][count*grid_h*grid_w] or NULL: s for allowed
 *              pairs, -inf elsewhere
 *   qmean_opt  fp32 [heads][Nq][128] or NULL: the q block means
 *   q_rot_opt  bf16, q_tok's layout, or NULL; only with p->rope (else
 *              LCSA_ERR_INVALID_ARG): receives q rotated (the values the
 *              block means sum), so that lcsa_attention can read it with
 *              rope.base = 0 instead of rotating q again.  16-byte aligned, not
 *              overlapping q_tok.
 * Allowed candidates per row must not exceed LCSA_MAX_CANDIDATES.
 */
int lcsa_draft_mask(const lcsa_params *p, const void *q_tok, const lcsa_kv_cache *cache,
                    int32_t *kept_idx, int32_t *kept_cnt, float *scores_opt,
                    float *qmean_opt, void *q_rot_opt, int32_t *d_status, void *stream);

/*
 * lcsa_attention - block_sparse_attn_func of learn.html 2.2 (reading notes
 * 关键设计 2): for every query token of block i, exact
 * softmax(q k^T * scale) V over the 128 tokens of each kept key block of row
 * (h, i) and nothing else; online softmax with fp32 accumulation, bf16
 * tensor-core products.
 *   q_tok    bf16 token layout [heads][2*q_layers][8*grid_h][8*grid_w][128]
 *   kept_idx int32 [heads][Nq][topk], kept_cnt int32 [heads][Nq]: the first
 *            kept_cnt entries of a row are used (any order, no duplicates)
 *   out_tok  bf16, same layout as q_tok (written; may not alias q_tok)
 *   lse_opt  fp32 [heads][2*q_layers][8*grid_h][8*grid_w] or NULL: natural
 *            log of the softmax denominator of each query token
 * With p->rope, the Q tiles are rotated (lcsa_rope) before the products (the
 * keys were rotated by the cache append).  That rotation runs inside the
 * kernel on every Q tile; the faster path, when lcsa_draft_mask runs first,
 * is its q_rot_opt copy passed here as q_tok with rope.base = 0: the same
 * rotated values, bit for bit, and no rotation left in this kernel.
 * A row with kept_cnt == 0 gets zeros (lse -inf).  A kept index outside
 * [0, count*grid_h*grid_w) or a count outside [0, topk] sets
 * LCSA_ERR_BAD_INDEX and the row is written as if it kept nothing.
 */
int lcsa_attention(const lcsa_params *p, const void *q_tok, const lcsa_kv_cache *cache,
                   const int32_t *kept_idx, const int32_t *kept_cnt, void *out_tok,
                   float *lse_opt, int32_t *d_status, void *stream);

/*
 * lcsa_segment_mask - kept lists of the segment-masked dense attention of the
 * reading notes' Stage-1 teacher (关键设计 1, the alpha_ij equation): over a
 * packed sequence of segments (each one clip: a video, or an image as a
 * single-frame video) every token attends to every token of its own segment
 * and to no other.  The sequence is cut into 128-token tiles and segment s is
 * the seg_tiles[s] tiles after those of segments 0 .. s-1 (so every segment
 * holds a whole number of tiles, 128 * seg_tiles[s] tokens).  For every head
 * h and query tile i of segment s it writes
 *   kept_idx[h][i][0 .. n_s) = the segment's tiles in ascending order, then -1
 *                             up to topk,   kept_cnt[h][i] = n_s = seg_tiles[s].
 *   seg_tiles  HOST int32 [n_seg], each in [1, topk]; 1 <= n_seg <= LCSA_MAX_SEGMENTS
 *   kept_idx   device int32 [heads][tiles][topk], kept_cnt device int32 [heads][tiles],
 *              tiles = sum of seg_tiles; both 4-byte aligned
 * lcsa_attention then computes the masked attention exactly: with q, k, v the
 * packed sequence as bf16 [heads][128 * tiles][128] (the token layout with
 * grid_h = grid_w = 1: a tile is one block-layer), k and v appended as
 * `tiles` layers to a cache of grid 1 x 1, and params {grid 1 x 1,
 * q_layers = tiles, topk}.  Asynchronous on `stream`; returns
 * LCSA_ERR_INVALID_ARG (nothing enqueued) for a bad table or size.
 */
int lcsa_segment_mask(const int32_t *seg_tiles, int32_t n_seg, int32_t heads, int32_t topk, int32_t *kept_idx,
                      int32_t *kept_cnt, void *stream);

/* Human-readable name of a status code or of a device status word. */
const char *lcsa_status_string(int code);

/* Library ABI version (major * 100 + minor). */
int lcsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LCSA_H */
