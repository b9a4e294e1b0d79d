/*
 * mmdit.h -- C ABI of the joint video/audio attention hot path (sm_100a).
 *
 * The library implements the attention layer of a dual-stream MMDiT video +
 * audio diffusion transformer as described for SkyReels-V4:
 *   - "SkyReels-V4: Multi-modal Video-Audio Generation, Inpainting and
 *     Editing model" (Chinese digest of arXiv 2602.21818), workflow steps 1-3
 *     and novelties 4-5;
 *   - "SkyReels-V4: dual-stream MMDiT ..." (trdm.cn blog), sections 2.1-2.2;
 * plus an optional block-sparse mode after
 *   - "Prism: dynamic sparse attention for native 2K joint video-audio
 *     generation" (reading guide of arXiv 2610.05416), Method section 3.
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors are BSHD: element (b, n, h, c) of a tensor described by
 * mmdit_tensor_desc d sits at  b*d.stride_batch + n*d.stride_tok + h*d.head_dim + c
 * elements from the base pointer (heads are packed, channels contiguous).
 * Strides are in elements; for bf16 tensors stride_tok*2 and stride_batch*2
 * must be multiples of 16 bytes and the base pointer 16-byte aligned.
 *
 * Ownership: every pointer is caller-owned device memory (except the
 * descriptor / layout structs, which are host memory read during the call).
 * The library never allocates device memory on these calls: scratch comes
 * from the caller's `workspace`, sized by the matching *_workspace_size query.
 *
 * Streams: every call only enqueues work on `stream` (a cudaStream_t; NULL is
 * the legacy default stream) and returns without synchronising.
 *
 * Errors: calls return an mmdit_status.  Arguments are validated before any
 * launch; on error nothing is launched and mmdit_last_error() describes the
 * problem (thread-local string).  Device-side waits are bounded: a wait that
 * runs out records MMDIT_ETIMEOUT in a per-device flag, the kernel releases its
 * resources and returns; mmdit_device_status() reads and clears that flag.
 */
#ifndef MMDIT_H_
#define MMDIT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MMDIT_API __attribute__((visibility("default")))
#else
#define MMDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mmdit_stream_t; /* same type as cudaStream_t */

typedef enum {
  MMDIT_OK = 0,
  MMDIT_EINVAL = 1,       /* bad pointer, shape, stride, layout or parameter   */
  MMDIT_EUNSUPPORTED = 2, /* dtype / head_dim / architecture not supported     */
  MMDIT_EWORKSPACE = 3,   /* workspace missing or smaller than the size query  */
  MMDIT_ECUDA = 4,        /* a CUDA runtime/driver call failed                 */
  MMDIT_ETIMEOUT = 5,     /* a bounded device-side wait ran out                */
  MMDIT_EDEVCHECK = 6     /* a device-side index check failed (builds with the
                             device checks only; the access was skipped)        */
} mmdit_status;

enum { MMDIT_BF16 = 0, MMDIT_F32 = 1 };
enum { MMDIT_SEG_VIDEO = 0, MMDIT_SEG_AUDIO = 1, MMDIT_SEG_TEXT = 2 };
enum { MMDIT_ORDER_RASTER = 0, MMDIT_ORDER_BLOCK444 = 1 };
#define MMDIT_MAX_SEGMENTS 8

/*
 * One contiguous run of tokens in the per-batch-item sequence.  The sequence
 * of one batch item is the concatenation of the layout's segments; the usual
 * order is [conditioning frames | video | audio | text] but any order works.
 *
 *  kind = VIDEO: n_tokens = T*H*W latent tokens of T frames.  Token
 *      positions are (t0 + t, h, w).  Conditioning / reference latents are a
 *      video segment with t0 < 0 (SkyReels-V4 digest, step 1 and novelty 4:
 *      reference latents are concatenated along time with negative temporal
 *      indices).  order = RASTER stores tokens in (t, h, w) raster order;
 *      order = BLOCK444 stores them block-major: 4x4x4 blocks in (tb, hb, wb)
 *      raster order, tokens inside a block in (t, h, w) raster order over the
 *      block's real extent (short edge blocks hold only their real tokens).
 *  kind = AUDIO: token j has position (t0 + j*t_num/t_den, 0, 0).  With
 *      t_num/t_den = 21/218, 218 audio tokens span 21 latent frames
 *      (digest novelty 5; blog section 2.2).  T, H, W are ignored.
 *  kind = TEXT: position (0, 0, 0): the identity rotation.
 */
typedef struct {
  int32_t kind;
  int32_t n_tokens;
  int32_t T, H, W;
  int32_t t0;
  int32_t t_num, t_den;
  int32_t order;
} mmdit_segment;

typedef struct {
  int32_t n_seg;                          /* 1..MMDIT_MAX_SEGMENTS */
  mmdit_segment seg[MMDIT_MAX_SEGMENTS];  /* same for every batch item */
} mmdit_layout;

typedef struct {
  int32_t batch;      /* B >= 1 */
  int32_t n_tokens;   /* N >= 0 (tokens per batch item) */
  int32_t heads;      /* >= 1 */
  int32_t head_dim;   /* 128 (bf16 or f32) or 64 (f32 only) */
  int32_t dtype;      /* MMDIT_BF16 or MMDIT_F32 */
  int64_t stride_tok;   /* elements between consecutive tokens (>= heads*head_dim) */
  int64_t stride_batch; /* elements between consecutive batch items */
} mmdit_tensor_desc;

/* 3D RoPE parameters: theta and the channel split over the t / h / w axes
 * (dim_t + dim_h + dim_w = head_dim, each even).  44/42/42 at head_dim 128. */
typedef struct {
  float theta;
  int32_t dim_t, dim_h, dim_w;
} mmdit_rope_params;

/*
 * mmdit_rope_apply -- 3D RoPE over (t, h, w), in place on q and/or k.
 *   Digest novelty 4 (time-offset 3D RoPE) and 5 (audio scaling 21/218);
 *   blog section 2.2.  Channels are split into bands [t | h | w]; in band b of
 *   width d_b the interleaved pair (2i, 2i+1) (i counted from the band start)
 *   is rotated by angle pos_b * theta^(-2i/d_b).  Positions come from
 *   `layout` (never stored).
 *   q, k   : device [B, N, heads, head_dim] described by `desc`; either may be
 *            NULL (skipped), not both.  Updated in place.
 *   layout : segments must sum to desc->n_tokens.
 *   Errors : EINVAL (NULL both, bad layout/desc/bands), EUNSUPPORTED (dtype),
 *            ECUDA.
 */
MMDIT_API int mmdit_rope_apply(void* q, void* k, const mmdit_tensor_desc* desc,
                     const mmdit_layout* layout, const mmdit_rope_params* rope,
                     mmdit_stream_t stream);

/*
 * mmdit_joint_attn -- joint self-attention over the whole concatenated
 *   sequence of each batch item: O = softmax(Q K^T * scale) V per (batch,
 *   head), no causal mask (digest step 3; blog section 2.1: video/audio and
 *   text tokens attend jointly in one softmax, in both the dual-stream and the
 *   single-stream blocks).
 *   q, k, v, o : device [B, N, heads, head_dim], all described by `desc`
 *                (o may not alias q, k or v).
 *   lse        : NULL or device float [B, heads, N]: natural-log sum of exp of
 *                the scaled scores of each query row.
 *   rope_q     : NULL, or RoPE parameters to rotate Q by `layout` positions as
 *                it is loaded (K must then already be rotated, e.g. by
 *                mmdit_rope_apply with q = NULL).  bf16 only.
 *   cond_mask  : NULL or device uint8 [B, F, H, W] with F the frames of all
 *                video segments; the binary channel-concat mask M of digest
 *                step 2.  It is an input channel of the patch embedding, not an
 *                attention mask: it is shape-checked (mask_elems must equal
 *                B*F*H*W) and never read or applied.
 *   workspace  : may be NULL; mmdit_joint_attn_workspace_size() returns 0.
 *   Errors     : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_joint_attn(const void* q, const void* k, const void* v, void* o, float* lse,
                     const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                     float scale, const mmdit_rope_params* rope_q,
                     const uint8_t* cond_mask, int64_t mask_elems,
                     void* workspace, size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_joint_attn_workspace_size(const mmdit_tensor_desc* desc);

/*
 * mmdit_av_cross_attn -- bidirectional audio<->video cross-attention (digest
 *   step 3; blog section 2.2), both directions in one call:
 *     o_video = softmax(qv ka^T * scale) va     (video queries, audio keys)
 *     o_audio = softmax(qa kv^T * scale) vv     (audio queries, video keys)
 *   qv, kv, vv, o_video : device, described by `video` (N = video tokens,
 *                         conditioning frames included)
 *   qa, ka, va, o_audio : device, described by `audio`
 *   Both descriptors must agree on batch, heads, head_dim and dtype.  Inputs
 *   are expected to be RoPE-rotated already.  The audio-query direction
 *   splits the video keys across CTAs and merges partial results through the
 *   workspace (size from mmdit_av_cross_attn_workspace_size).
 *   Errors : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_av_cross_attn(const void* qv, const void* kv, const void* vv,
                        const void* qa, const void* ka, const void* va,
                        void* o_video, void* o_audio,
                        const mmdit_tensor_desc* video, const mmdit_tensor_desc* audio,
                        float scale, void* workspace, size_t ws_bytes,
                        mmdit_stream_t stream);
MMDIT_API size_t mmdit_av_cross_attn_workspace_size(const mmdit_tensor_desc* video,
                                          const mmdit_tensor_desc* audio);

/*
 * mmdit_text_cross_attn -- reinforced text cross-attention (digest step 3:
 *   in every layer the video tokens query the text embedding, beside the
 *   bidirectional audio<->video cross-attention):
 *     o_video = softmax(qv kt^T * scale) vt     (video queries, text keys)
 *   qv, o_video : device, described by `video` (N = video tokens, conditioning
 *                 frames included); o_video may not alias qv
 *   kt, vt      : device, described by `text` (N = text tokens, >= 1)
 *   Both descriptors must agree on batch, heads, head_dim and dtype.  Inputs
 *   are expected to be RoPE-rotated already (text tokens sit at position
 *   (0, 0, 0), where the rotation is the identity).  No workspace.
 *   Errors : EINVAL, EUNSUPPORTED, ECUDA.
 */
MMDIT_API int mmdit_text_cross_attn(const void* qv, const void* kt, const void* vt, void* o_video,
                          const mmdit_tensor_desc* video, const mmdit_tensor_desc* text,
                          float scale, mmdit_stream_t stream);

/*
 * mmdit_masked_joint_attn -- mask-guided region-restricted attention of the
 *   Refiner (blog section 4.2: with a spatial mask, only the target region is
 *   refined): for every video token whose mask value is non-zero, its row of
 *   O = softmax(Q K^T * scale) V over all tokens of its batch item (as in
 *   mmdit_joint_attn); every other row of o is left as it was.
 *   q, k, v, o : device [B, N, heads, 128] bf16 described by `desc`, Q and K
 *                already rotated (o may not alias q, k or v).
 *   layout     : segment table; video segments in raster order, all with the
 *                same H and W.
 *   mask       : device uint8 [B, F, H, W], F = frames of all video segments
 *                in sequence order (the binary mask M of digest step 2);
 *                mask_elems must equal B*F*H*W (0 and NULL allowed when the
 *                layout has no video token).
 *   workspace  : mmdit_masked_joint_attn_workspace_size(desc, layout) bytes,
 *                256-byte aligned: the row lists and compact copies of the
 *                masked Q and O rows (sized for every video token, since the
 *                count is only known on the device).
 *   Errors     : EINVAL, EUNSUPPORTED (fp32, block-major video), EWORKSPACE,
 *                ECUDA.
 */
MMDIT_API int mmdit_masked_joint_attn(const void* q, const void* k, const void* v, void* o,
                            const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                            float scale, const uint8_t* mask, int64_t mask_elems,
                            void* workspace, size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_masked_joint_attn_workspace_size(const mmdit_tensor_desc* desc,
                                              const mmdit_layout* layout);

/*
 * mmdit_flow_noise -- flow-matching input and target of one stream (digest
 *   step 4: z_t = t z_0 + (1 - t) eps, and the model is trained to predict the
 *   velocity z_0 - eps), fused in one elementwise pass:
 *     zt[b, i] = t[b] * z0[b, i] + (1 - t[b]) * eps[b, i]
 *     u[b, i]  = z0[b, i] - eps[b, i]
 *   for i < n of every batch item b < batch; math in fp32.
 *   z0, eps   : device, batch items (1..65535) of n values `stride` elements
 *               apart (stride >= n); the noise is an input, drawn by the caller.
 *   t         : device float [batch], the flow time of each item.
 *   zt, u     : device outputs with the same shape and stride; either may be
 *               NULL (not written), not both.
 *   dtype     : MMDIT_BF16 or MMDIT_F32 for all of z0, eps, zt, u.
 *   Pointers must be 16-byte aligned and stride * element size a multiple of
 *   16 bytes.  The video and the audio stream are separate calls.
 *   Errors : EINVAL, EUNSUPPORTED, ECUDA.
 */
MMDIT_API int mmdit_flow_noise(const void* z0, const void* eps, const float* t, void* zt, void* u,
                     int32_t batch, int64_t n, int64_t stride, int32_t dtype,
                     mmdit_stream_t stream);

/*
 * mmdit_flow_loss -- the flow-matching loss term of one stream (digest step 4:
 *   || v_theta - (z_0 - eps) ||^2), per batch item:
 *     loss[b] = sum over i < n of (v[b, i] - (z0[b, i] - eps[b, i]))^2
 *   in fp32, summed in a fixed order (the same bits on every call).  The
 *   layer's loss is the batch mean of loss_video[b] + loss_audio[b].
 *   v, z0, eps : device, same shape, stride and dtype rules as mmdit_flow_noise
 *   loss       : device float [batch] output
 *   workspace  : mmdit_flow_loss_workspace_size(batch, n) bytes, 256-byte
 *                aligned (per-block partial sums).
 *   Errors : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_flow_loss(const void* v, const void* z0, const void* eps, float* loss,
                    int32_t batch, int64_t n, int64_t stride, int32_t dtype, void* workspace,
                    size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_flow_loss_workspace_size(int32_t batch, int64_t n);

/*
 * mmdit_av_cross_attn_noalloc -- the same cross-attention as
 *   mmdit_av_cross_attn, for callers that cannot allocate device memory or
 *   size a workspace (a plugin inside a runtime that owns every device
 *   allocation, a serving loop that forbids allocation after start-up).  The
 *   source pages have no counterpart: this is an interface convenience.
 *   Scratch is a fixed file-scope device array of MMDIT_NOALLOC_SCRATCH_BYTES
 *   that every GPU loading the library holds until exit; the call performs no
 *   cudaMalloc/cudaFree and no allocating library routine.  Arguments and
 *   outputs are those of mmdit_av_cross_attn minus the workspace; bf16 only.
 *   The first call on each device (with that device current) looks up the
 *   array's device address and caches it, so make that first call before any
 *   stream capture.  All calls share the array: calls that overlap on the GPU
 *   race.  The split of the video keys is reduced until the partial results
 *   fit; problems whose batch*heads*ceil(Na/256)*256 rows need more than the
 *   array even unsplit (130 floats per row) are rejected with MMDIT_EINVAL.
 *   Errors : EINVAL, EUNSUPPORTED, ECUDA.
 */
#define MMDIT_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
MMDIT_API int mmdit_av_cross_attn_noalloc(const void* qv, const void* kv, const void* vv,
                                          const void* qa, const void* ka, const void* va,
                                          void* o_video, void* o_audio,
                                          const mmdit_tensor_desc* video,
                                          const mmdit_tensor_desc* audio, float scale,
                                          mmdit_stream_t stream);

/*
 * mmdit_block_select -- hybrid top-k / top-p key-block selection of the
 *   block-sparse mode (Prism guide, Method section 3).
 *   Q and K of one block-major video segment are mean-pooled per 4x4x4 block
 *   (fp32, over each block's real tokens) into Qbar, Kbar.  For query block i
 *   of each (batch, head): P_i = softmax_j(Qbar_i . Kbar_j * scale), and
 *   S_i = TopK(P_i, top_k) U TopP(P_i, top_p), where blocks are ranked by P
 *   descending (ties: lower block id first), TopK is the first min(top_k, n)
 *   blocks and TopP the shortest prefix whose cumulative probability reaches
 *   top_p (the crossing block included; all blocks if it never does).
 *   q, k      : device [B, N, heads, 128] bf16, N = the video segment's tokens
 *   layout    : exactly one VIDEO segment with order BLOCK444
 *   cap       : row capacity of block_idx; must be >= the number of blocks
 *               (a list is never truncated)
 *   block_idx : device int32 [B, heads, nblocks, cap]: S_i in ascending block
 *               id, entries past block_cnt are left unwritten
 *   block_cnt : device int32 [B, heads, nblocks]: |S_i|
 *   workspace : size from mmdit_block_select_workspace_size (pooled blocks)
 *   Errors    : EINVAL (layout, cap, top_k < 0, top_p outside [0, 1]),
 *               EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_block_select(const void* q, const void* k, const mmdit_tensor_desc* desc,
                       const mmdit_layout* layout, int top_k, float top_p, float scale,
                       int cap, int32_t* block_idx, int32_t* block_cnt,
                       void* workspace, size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_block_select_workspace_size(const mmdit_tensor_desc* desc,
                                         const mmdit_layout* layout);

/*
 * mmdit_sparse_attn -- attention restricted to selected key blocks (Prism
 *   guide, Method section 3: online-softmax attention over S_i only).  Every
 *   token of query block i attends, in one softmax, to the tokens of the key
 *   blocks listed in block_idx[b, h, i, 0:block_cnt[b, h, i]].
 *   q, k, v, o : device [B, N, heads, 128] bf16, block-major video segment
 *   block_idx, block_cnt : as written by mmdit_block_select (ids must be
 *               ascending and < nblocks; counts in [0, nblocks]); a query block
 *               with an empty list gets a zero output row
 *   workspace  : size from mmdit_sparse_attn_workspace_size (per-CTA merged
 *               block lists)
 *   Errors     : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_sparse_attn(const void* q, const void* k, const void* v, void* o,
                      const mmdit_tensor_desc* desc, const mmdit_layout* layout,
                      const int32_t* block_idx, const int32_t* block_cnt, int cap,
                      float scale, void* workspace, size_t ws_bytes,
                      mmdit_stream_t stream);
MMDIT_API size_t mmdit_sparse_attn_workspace_size(const mmdit_tensor_desc* desc,
                                        const mmdit_layout* layout, int cap);

/*
 * mmdit_av_cross_attn_norms -- mmdit_av_cross_attn plus the output norm of
 *   every video token of the video-query (audio -> video) direction:
 *     video_norm[b, n] = || o_video[b, n, :, :] ||_2  over all heads and channels
 *   (the norms a_{t,h,w} the Prism guide's Method section 1 caches from one
 *   layer to guide the content-adaptive block shapes of the next; computed
 *   from the fp32 output rows before their bf16 rounding, summed over heads in
 *   a fixed order).  Other arguments as mmdit_av_cross_attn (bf16 only);
 *   video_norm : device float [B, N_video].
 *   workspace  : mmdit_av_cross_attn_norms_workspace_size bytes, 256-byte
 *                aligned (the cross-attention partials + per-head norms).
 *   Errors : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_av_cross_attn_norms(const void* qv, const void* kv, const void* vv,
                                        const void* qa, const void* ka, const void* va,
                                        void* o_video, void* o_audio,
                                        const mmdit_tensor_desc* video,
                                        const mmdit_tensor_desc* audio, float scale,
                                        float* video_norm, void* workspace, size_t ws_bytes,
                                        mmdit_stream_t stream);
MMDIT_API size_t mmdit_av_cross_attn_norms_workspace_size(const mmdit_tensor_desc* video,
                                                          const mmdit_tensor_desc* audio);

/*
 * Content-adaptive block shapes (Prism guide, Key ideas and Method sections
 * 1-2).  A raster-order video (T x H x W tokens per batch item) is cut into
 * 8 x 8 x 8 macro-zones (short at the far edges).  Per zone m, from the value
 * features V (all heads and channels, D = heads x 128):
 *   sigma^2_{v,d}(m) = (1/D) sum_c (1/Z_d) sum_i (Vbar^(d)_{m,i,c} - mu^(d)_{m,c})^2
 * (Vbar^(d)_{m,i}: mean of V over the zone's tokens with index i along axis
 * d; mu^(d): the mean of those), r_{v,d} = sigma^2_{v,d} / sum_d' sigma^2_{v,d'};
 * from the A->V cross-attention output norms a of the preceding layer,
 * abar(m) = the zone mean of a / the largest zone mean, and vhat_{a,d}(m) =
 * the directional variance of a normalised like r;
 *   g_d(m) = r_{v,d}(m) + abar(m) vhat_{a,d}(m) + eps.
 * The density rho(m) = sum_d sigma^2_{v,d}(m) / its largest value over the
 * zones picks the block volume B(m) = 64 (rho >= tau_128), 128 (rho >=
 * tau_256) or 256; the block shape is the candidate of that volume nearest in
 * log2 space to l*_d = -1/2 log2 g_d + 1/3 (log2 B + 1/2 sum_d' log2 g_d').
 * Candidates: edges 2, 4 or 8 with product B, 16 shapes, numbered
 *   0..6   (B = 64):  (2,4,8) (2,8,4) (4,2,8) (4,4,4) (4,8,2) (8,2,4) (8,4,2)
 *   7..12  (B = 128): (2,8,8) (4,4,8) (4,8,4) (8,2,8) (8,4,4) (8,8,2)
 *   13..15 (B = 256): (4,8,8) (8,4,8) (8,8,4)
 * as (b_T, b_H, b_W); distance ties go to the lower number.  A zone is cut
 * into blocks of its shape (clipped at the zone edge).  Adaptive storage
 * order: zones in raster order, each zone's blocks in raster order, each
 * block's tokens in (t, h, w) raster order -- every block is one contiguous
 * run of tokens, so the block-table calls below attend over it directly.
 * The choices the guide leaves open (the 16 shapes, rho, the normalisations
 * of abar and vhat, eps, short zones) are the readings stated above.
 */
typedef struct {
  float tau_128;  /* rho threshold of B = 64 vs 128 (0.5) */
  float tau_256;  /* rho threshold of B = 128 vs 256 (0.25) */
  float eps;      /* epsilon of g_d (1e-6) */
} mmdit_adaptive_params;

/* Macro-zones of a T x H x W video, and the block-table capacity a plan of it
 * may need (8 per zone: the finest volume, 64 tokens, in a full zone). */
MMDIT_API int mmdit_adaptive_num_zones(int T, int H, int W);
MMDIT_API int mmdit_adaptive_max_blocks(int T, int H, int W);

/*
 * mmdit_adaptive_plan -- the content-adaptive partition of every batch item.
 *   v          : device bf16 [B, N, heads, 128], N = T*H*W, raster order (the
 *                value features of the layer)
 *   a_norm     : NULL (no audio guidance: abar = 0), or device float [B, N]:
 *                the A->V output norms of the preceding layer (as written by
 *                mmdit_av_cross_attn_norms), raster order
 *   params     : NULL for (0.5, 0.25, 1e-6), else 0 <= tau_256 <= tau_128 <= 1
 *                and eps > 0
 *   zones      : device int32 [B, n_zones, 4], 16-byte aligned: per zone
 *                {shape number 0..15, first storage position, first block,
 *                blocks}
 *   blocks     : device int32 [B, max_blocks, 2]: {start, length} of every
 *                block in the adaptive storage order; n_blocks: device int32
 *                [B] (entries past n_blocks[b] are not written)
 *   max_blocks : >= mmdit_adaptive_max_blocks(T, H, W), <= 6000
 *   workspace  : mmdit_adaptive_plan_workspace_size bytes, 256-byte aligned
 *   The statistics are fp32 sums of the bf16 values; the plan arithmetic is
 *   fp64.  Errors : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_adaptive_plan(const void* v, const float* a_norm,
                                  const mmdit_tensor_desc* desc, int T, int H, int W,
                                  const mmdit_adaptive_params* params, int32_t* zones,
                                  int32_t* blocks, int32_t* n_blocks, int max_blocks,
                                  void* workspace, size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_adaptive_plan_workspace_size(const mmdit_tensor_desc* desc, int T, int H,
                                                    int W);

/*
 * mmdit_adaptive_permute -- moves token rows between raster order and the
 *   adaptive storage order of a plan: inverse = 0 writes dst[s(t,h,w)] =
 *   src[(t H + h) W + w], inverse = 1 the reverse.  Up to three tensors (e.g.
 *   Q, K, V) in one call; src[i] and dst[i] are device [B, N, heads, 128] bf16
 *   described by `desc` (N = T*H*W), dst[i] may not alias src[i].  zones is a
 *   plan's zone table.  Errors : EINVAL, EUNSUPPORTED, ECUDA.
 */
MMDIT_API int mmdit_adaptive_permute(const void* const* src, void* const* dst, int n_tensors,
                                     const mmdit_tensor_desc* desc, int T, int H, int W,
                                     const int32_t* zones, int inverse, mmdit_stream_t stream);

/*
 * mmdit_block_select_table / mmdit_sparse_attn_table -- mmdit_block_select and
 *   mmdit_sparse_attn over the blocks of a block table (Prism guide, Method
 *   section 3) instead of the 4x4x4 blocks of a grid: per batch item b the
 *   blocks are blocks[b, i] = {start, length}, i < n_blocks[b] (device int32,
 *   as written by mmdit_adaptive_plan), consecutive runs of 1..256 tokens of
 *   q, k, v, o, which hold the video in that block storage order.  Block ids
 *   index the table; block_idx is [B, heads, max_blocks, cap], block_cnt
 *   [B, heads, max_blocks], cap >= max_blocks.  Selection and attention are
 *   those of the 4x4x4 calls (pooled means over each block's tokens, P_i,
 *   S_i = TopK U TopP, attention of every token of query block i over the
 *   tokens of S_i).  A table entry outside [0, N) or longer than 256 tokens
 *   is treated as an empty block.
 *   Errors : EINVAL, EUNSUPPORTED, EWORKSPACE, ECUDA.
 */
MMDIT_API int mmdit_block_select_table(const void* q, const void* k, const mmdit_tensor_desc* desc,
                                       const int32_t* blocks, const int32_t* n_blocks,
                                       int max_blocks, int top_k, float top_p, float scale,
                                       int cap, int32_t* block_idx, int32_t* block_cnt,
                                       void* workspace, size_t ws_bytes, mmdit_stream_t stream);
MMDIT_API size_t mmdit_block_select_table_workspace_size(const mmdit_tensor_desc* desc,
                                                         int max_blocks);
MMDIT_API int mmdit_sparse_attn_table(const void* q, const void* k, const void* v, void* o,
                                      const mmdit_tensor_desc* desc, const int32_t* blocks,
                                      const int32_t* n_blocks, int max_blocks,
                                      const int32_t* block_idx, const int32_t* block_cnt, int cap,
                                      float scale, void* workspace, size_t ws_bytes,
                                      mmdit_stream_t stream);
MMDIT_API size_t mmdit_sparse_attn_table_workspace_size(const mmdit_tensor_desc* desc,
                                                        int max_blocks);

/* Number of 4x4x4 blocks of the single BLOCK444 video segment of `layout`
 * (0 if the layout is not a single such segment). */
MMDIT_API int mmdit_num_blocks(const mmdit_layout* layout);

/* Reads and clears the device error flag of the current device after
 * synchronising `stream`: MMDIT_OK, or MMDIT_ETIMEOUT if a bounded wait ran out
 * in a kernel since the last call, or MMDIT_EDEVCHECK if a device-side index
 * check of the checked build failed, or MMDIT_ECUDA.  While the flag is set,
 * the library's attention kernels skip their work. */
MMDIT_API int mmdit_device_status(mmdit_stream_t stream);

/* Diagnostic, no counterpart on the source pages: launches one warp that
 * waits on an mbarrier nothing ever arrives at, through the library's bounded
 * device wait, with a limit of limit_ms (1..2000).  The wait gives up, records
 * MMDIT_ETIMEOUT in the device error word (read and cleared by
 * mmdit_device_status; until then the library's attention kernels skip their
 * work) and writes 1 to the device int *waited_out.  Exercises failure
 * detection without faulting or hanging the GPU.  Errors: EINVAL, ECUDA. */
MMDIT_API int mmdit_selftest_wait_timeout(int limit_ms, int* waited_out, mmdit_stream_t stream);

/* Thread-local description of the last error returned on this thread. */
MMDIT_API const char* mmdit_last_error(void);

/* Library version string. */
MMDIT_API const char* mmdit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MMDIT_H_ */
