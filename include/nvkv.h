/*
 * nvkv.h -- C ABI of the NVFP4 KV-cache append and block-causal chunk
 * attention library for B200 (sm_100a).
 *
 * The path it implements, per autoregressive (AR) step of a streaming video
 * diffusion generator:
 *
 *   kv_ring_evict            drop the oldest non-sink frames when the ring is full
 *   nvfp4_kv_append          quantize the new chunk's K/V to NVFP4 and write it,
 *                            in place, into free frame slots of the cache
 *   chunk_attention_nvfp4kv  the chunk's queries attend over the dequantized,
 *                            RoPE-rotated sink + window K/V
 *
 * plus a bf16-KV twin of the cache (bf16_kv_append, chunk_attention_bf16kv).
 *
 * Sources: "NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
 * generation" (hysenlabs.com), section "NVFP4, sequence parallel and the async
 * decode path": the KV cache is kept in the same NVFP4 format as the W4A4
 * generator, beside a BF16 path; the listed optimisations are in-place
 * quantized KV-cache updates, faster FP4 KV dequantization, fused RoPE and
 * reduced KV-cache synchronisation; attention sinks keep the streaming
 * generator from drifting and extend to multi-shot video.  "NVlabs LongLive"
 * (refft.com), Core Analysis block "How do KV-cache relative RoPE and
 * TriAttention work together": RoPE is applied relative to the cache, so new
 * chunks append without position drift.  "LongLive: NVIDIA long video
 * generation" (evermx.com), heading "Multi-Shot Generation": shots attend to
 * relevant past context without bleeding across cuts.
 *
 * NVFP4 format used by the cache (the workload contract of the tiny reference
 * case): per 16 contiguous head_dim elements one E4M3 block scale
 *   s_b = E4M3_RNE(min(fl32(amax16 / fl32(6 * s_g)), 448)),
 * E2M1 codes q = E2M1_RNE_sat(fl32(x / fl32(s_b * s_g))) (a magnitude that
 * rounds to zero is stored as code 0; s_b = 0 gives all-zero codes), two codes
 * per byte with element 2i in the low nibble, and one FP32 global scale per
 * (K or V, batch, head) fixed by the first chunk: s_g = fl32(amax / 2688)
 * (1 when that is zero or not a normal float).  Dequantized value:
 * e2m1(q) * s_b * s_g.
 *
 * Conventions
 *  - All device memory is allocated by the caller, once, with the sizes
 *    nvkv_plane_bytes() and nvkv_attention_workspace_bytes() report.  The
 *    library never allocates, frees or synchronises; every device call is
 *    asynchronous and ordered on the stream it is given.
 *  - Host validation errors are returned before anything is launched and leave
 *    the ring unchanged.  A launch failure returns NVKV_ERR_CUDA.  Errors found
 *    on the device (a pipeline wait that ran out of its bound) are written to
 *    cache->status as an nvkv_status value; the caller reads it after a sync.
 *  - q, k, v and out are contiguous bf16 tensors [B][Lq][H][128] with
 *    Lq = C * T tokens (C frames of T = grid_h * grid_w tokens, token t of a
 *    frame at row t / grid_w, column t % grid_w).  Device pointers must be
 *    16-byte aligned.
 *  - The ring (nvkv_ring) is a host-side value owned by the caller.  Kernels
 *    receive a snapshot of it as a launch parameter: no host-to-device copy and
 *    no host sync per step.
 */
#ifndef NVKV_H
#define NVKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NVKV_API __attribute__((visibility("default")))
#else
#define NVKV_API
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *nvkv_stream;

typedef enum {
    NVKV_OK = 0,
    NVKV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad shot id          */
    NVKV_ERR_UNSUPPORTED = 2,  /* head_dim != 128, limits exceeded, no sm_100  */
    NVKV_ERR_ALIGNMENT = 3,    /* a device pointer is not 16-byte aligned      */
    NVKV_ERR_CAPACITY = 4,     /* no room for the chunk (evict first) or too
                                  few evictable frames; workspace too small    */
    NVKV_ERR_STATE = 5,        /* bad magic/version, ring does not match desc,
                                  attention before any append, wrong kv dtype  */
    NVKV_ERR_CUDA = 6,         /* a CUDA launch failed                         */
    NVKV_ERR_TIMEOUT = 7       /* device status only: a bounded wait expired   */
} nvkv_status;

#define NVKV_MAGIC 0x4E564B56u /* "NVKV" */
#define NVKV_VERSION 2u
#define NVKV_HEAD_DIM 128
#define NVKV_MAX_BATCH 16
#define NVKV_MAX_FRAMES 64     /* S + W */
#define NVKV_MAX_CHUNK 16      /* C */
#define NVKV_MAX_SHARDS 16     /* shard_count, and parts of one nvkv_lse_merge */

enum { NVKV_KV_NVFP4 = 0, NVKV_KV_BF16 = 1 };

/* Problem description (a value type; fill it with nvkv_desc_init). */
typedef struct {
    uint32_t magic, version;
    int32_t B;            /* batch (independent streams)                       */
    int32_t H;            /* heads                                             */
    int32_t D;            /* head_dim, must be 128                             */
    int32_t grid_h;       /* latent rows per frame                             */
    int32_t grid_w;       /* latent columns per frame; T = grid_h * grid_w      */
    int32_t C;            /* frames per chunk (per AR step)                    */
    int32_t S;            /* sink frames (the first S frames ever appended)     */
    int32_t W;            /* window frames, the current chunk included          */
    int32_t kv_dtype;     /* NVKV_KV_NVFP4 or NVKV_KV_BF16                      */
    float rope_base;      /* 10000                                             */
    int32_t rope_split[3];/* head_dim channels for (frame, h, w): 44, 42, 42    */
    int32_t shard_rank;   /* sequence-parallel KV split (nvkv_desc_set_shard): */
    int32_t shard_count;  /* this cache holds tokens [rank*T/count,
                             (rank+1)*T/count) of every frame; 0 of 1 = all   */
} nvkv_desc;

/* Device planes of one cache (caller-owned; sizes from nvkv_plane_bytes).
 * Ts = T / shard_count tokens of each frame are cached, in Tr = Ts rounded up
 * to even rows per frame slot (an odd Ts adds one padding row, so that every
 * slot's scale rows start on a 16-byte boundary); R = (S + W) * Tr rows per
 * (batch, head).  Physical frame slot p holds rows [p*Tr, p*Tr + Ts), row
 * p*Tr + i being token shard_rank*Ts + i of the frame in that slot; the
 * padding row is never written, and no result depends on its contents.
 *   NVFP4: k_data/v_data = codes [B][H][R][64] u8, k_scales/v_scales = E4M3
 *          block scales [B][H][R][8] u8, amax [2][B][H] (float bits, K then
 *          V), s_g [2][B][H] f32.
 *   BF16:  k_data/v_data = [B][H][R][128] bf16; the other planes may be NULL.
 * status: one int32, cleared by the caller; device errors are written here. */
typedef struct {
    void *k_data, *v_data;
    void *k_scales, *v_scales;
    uint32_t *amax;
    float *s_g;
    int32_t *status;
} nvkv_cache;

enum {
    NVKV_PLANE_K_DATA = 0, NVKV_PLANE_V_DATA = 1, NVKV_PLANE_K_SCALES = 2,
    NVKV_PLANE_V_SCALES = 3, NVKV_PLANE_AMAX = 4, NVKV_PLANE_SCALE_G = 5,
    NVKV_PLANE_STATUS = 6
};

/* Frame flags in the ring. */
#define NVKV_FRAME_SINK 1u       /* global attention sink, never evicted        */
#define NVKV_FRAME_PINNED 2u     /* per-shot sink of the running shot           */
#define NVKV_FRAME_SHOT_LAST 4u  /* last frame of a shot that has ended          */

/* Ring state of one stream.  Resident frames in logical order: sink frames
 * first, then the others by age.  The RoPE frame index of a resident frame is
 * its position in this order. */
typedef struct {
    int32_t n_resident;
    int32_t shot;                         /* running shot id                  */
    int32_t pin_next;                     /* next chunk is a per-shot sink    */
    int32_t n_appended;                   /* frames appended so far           */
    int32_t slot[NVKV_MAX_FRAMES];        /* logical index -> physical slot   */
    int32_t frame[NVKV_MAX_FRAMES];       /* logical index -> frame number    */
    int32_t frame_shot[NVKV_MAX_FRAMES];  /* logical index -> shot id         */
    uint32_t flags[NVKV_MAX_FRAMES];      /* NVKV_FRAME_*                     */
} nvkv_ring_stream;

typedef struct {
    uint32_t magic, version;
    int32_t B, capacity, C, S;            /* copied from the desc at init      */
    int32_t scales_fixed;                 /* 1 once step 1 fixed the s_g       */
    int32_t steps;                        /* appends so far                   */
    nvkv_ring_stream s[NVKV_MAX_BATCH];
} nvkv_ring;

/* Fill a desc with D = 128, RoPE split 44/42/42 and base 10000.  Returns
 * NVKV_ERR_INVALID_ARG / NVKV_ERR_UNSUPPORTED for shapes outside the limits
 * (B <= 16, S + W <= 64, 1 <= C <= min(W, 16), T >= 1, grid_h, grid_w < 65536). */
NVKV_API nvkv_status nvkv_desc_init(nvkv_desc *desc, int B, int H, int grid_h, int grid_w, int C, int S,
                           int W, int kv_dtype);

/* Sequence-parallel KV split ("NVlabs/LongLive 2.0: NVFP4 parallel
 * infrastructure for long video generation", section "NVFP4, sequence
 * parallel and the async decode path": sequence-parallel inference to cut the
 * KV memory each GPU holds).  Makes desc describe shard `rank` of `count`
 * caches that together hold the whole cache: shard r keeps tokens
 * [r*T/count, (r+1)*T/count) of every frame, so each holds 1/count of the K/V
 * and of the attention work.  The ring logic is unchanged: every shard runs
 * the same ring (same slots, same eviction) on the same calls.
 *  - The appends take the whole chunk's k, v ([B][C*T][H][128]) and write the
 *    shard's tokens; the first append measures amax over the whole chunk, so
 *    all shards fix the same s_g.
 *  - The attention calls take the whole chunk's q and return, for every
 *    query, the attention over the shard's keys only, with its lse; the
 *    shards' results are combined by nvkv_lse_merge.
 * NVKV_ERR_INVALID_ARG unless 1 <= count <= NVKV_MAX_SHARDS, 0 <= rank <
 * count and T is a multiple of count.  An odd T/count (1560 tokens in 8
 * shards: 195) is fine: the slots then carry a padding row.  count = 1 gives
 * back the whole cache. */
NVKV_API nvkv_status nvkv_desc_set_shard(nvkv_desc *desc, int rank, int count);

/* Bytes the caller must allocate for one plane (NVKV_PLANE_*) of a cache of
 * this desc; 0 for planes the dtype does not use or for an invalid desc. */
NVKV_API size_t nvkv_plane_bytes(const nvkv_desc *desc, int plane);

/* Empty ring for this desc (all frames free, shot 0). */
NVKV_API nvkv_status nvkv_ring_init(const nvkv_desc *desc, nvkv_ring *ring);

/* Host only, no device work: in every stream, drop the n_frames oldest
 * resident frames that are neither sink nor pinned (the sink + rolling window
 * rule: "eviction drops the oldest non-sink frame").  NVKV_ERR_CAPACITY, and
 * no change, if any stream has fewer evictable frames. */
NVKV_API nvkv_status kv_ring_evict(const nvkv_desc *desc, nvkv_ring *ring, int n_frames);

/* Host only: stream b starts shot shot_id (>= the running one; equal is a
 * no-op).  The newest resident frame is marked as its shot's last frame,
 * every pinned frame is unpinned, and the next chunk appended to b becomes the
 * new shot's per-shot sink (pinned until the following shot begins).  A chunk
 * of shot s sees the global sink, all frames of shot s and the last frame of
 * each earlier shot ("LongLive: NVIDIA long video generation", heading
 * "Multi-Shot Generation"). */
NVKV_API nvkv_status kv_ring_begin_shot(const nvkv_desc *desc, nvkv_ring *ring, int b, int shot_id);

/* Host query of what the newest chunk of stream b sees: for each visible frame
 * in logical order its physical slot, RoPE frame index and frame number
 * (arrays of at least NVKV_MAX_FRAMES entries, any may be NULL).  Returns the
 * number of visible frames, or -1 on a bad argument.  *query_pos0 (may be
 * NULL) receives the RoPE frame index of the newest chunk's first frame. */
NVKV_API int nvkv_ring_visible(const nvkv_desc *desc, const nvkv_ring *ring, int b, int32_t *slots,
                      int32_t *rope_pos, int32_t *frames, int32_t *query_pos0);

/* Host only: the ring update of one append without any device work.  Assigns
 * C free physical slots per stream (lowest free first), records the chunk's
 * frames as resident (sink flag for the first S frames ever appended, pinned
 * if the chunk opens a shot) and writes the slots to slots_out[b * C + c]
 * (may be NULL).  For callers that write a chunk's K/V into those slots with
 * their own kernel.  NVKV_ERR_CAPACITY (no change) if a stream has fewer than
 * C free frames. */
NVKV_API nvkv_status nvkv_ring_push_chunk(const nvkv_desc *desc, nvkv_ring *ring,
                                          int32_t *slots_out);

/* Quantize-append, in place.  k, v: device bf16 [B][Lq][H][128].  Assigns C
 * free physical slots per stream (lowest free first), quantizes K and V to
 * NVFP4 and writes codes and scales into those slots; on the first append it
 * also measures the per-(K/V, batch, head) amax of the chunk and fixes s_g.
 * NVKV_ERR_CAPACITY (no change) if a stream has fewer than C free frames. */
NVKV_API nvkv_status nvfp4_kv_append(const nvkv_desc *desc, const nvkv_cache *cache, nvkv_ring *ring,
                            const void *k, const void *v, nvkv_stream stream);

/* nvfp4_kv_append for callers that cannot allocate device memory (no
 * counterpart in the paper; an interface addition of this library).  The
 * regular call needs the small caller-allocated scratch plane cache->amax,
 * where the first append reduces each head's absolute maximum.  An
 * inference-engine plugin whose enqueue step may not allocate, or a process
 * whose device memory is all owned by another allocator, cannot provide it.
 * This call keeps that scratch in a fixed array inside the library's device
 * image instead (2 KiB; every GPU that loads the library holds it until the
 * process exits) and allocates nothing.  Same inputs, outputs, slot logic and
 * results as nvfp4_kv_append; cache->amax is ignored and may be NULL.
 *  - B * H must be <= 256, else NVKV_ERR_UNSUPPORTED.
 *  - The first call on a device sets up the array's address for that device
 *    (with that device current) and keeps it for the process; make it before
 *    any stream capture.  After a cudaDeviceReset of that device the kept
 *    address is stale: do not call this entry point on that device again.
 *  - All calls share the array: a scale-fixing first append clears it before
 *    use; calls whose work overlaps on the GPU race on it, so serialise them. */
NVKV_API nvkv_status nvfp4_kv_append_noalloc(const nvkv_desc *desc, const nvkv_cache *cache,
                                             nvkv_ring *ring, const void *k, const void *v,
                                             nvkv_stream stream);

/* Quantize-append for the block-scaled FP4 Q K^T reading (the KV cache "in
 * the same format" as the W4A4 generator: evermx.com, heading "NVFP4
 * Quantization End-to-End"; relative RoPE: "NVlabs LongLive", refft.com, Core
 * Analysis block on KV-cache relative RoPE).  As nvfp4_kv_append, but each K
 * row first has its spatial RoPE pairs (the 42-channel h and w segments)
 * rotated at its token's (h, w), in float: cos and sin of the fp64 angle
 * pos * rope_base^(-2i/42), each rounded once to float, and (fl(fl(x c) -
 * fl(y s)), fl(fl(x s) + fl(y c))); the frame segment stays unrotated and V
 * is appended as usual.  The first chunk's K amax is taken over the rotated
 * rows.  The cache this fills holds keys for a contraction that applies only
 * the frame rotation at read time; chunk_attention_nvfp4kv, which rotates
 * the cached keys in all three segments, does not read it.
 * NVKV_ERR_UNSUPPORTED unless the RoPE split is 44/42/42 and grid_h, grid_w
 * <= 90; otherwise as nvfp4_kv_append. */
NVKV_API nvkv_status nvfp4_kv_append_spatial_rope(const nvkv_desc *desc, const nvkv_cache *cache,
                                                  nvkv_ring *ring, const void *k, const void *v,
                                                  nvkv_stream stream);

/* The query side of the same reading: every row of the chunk's Q quantized
 * to NVFP4 once per visible key frame.  For the frame at RoPE index f_k
 * (visible frame j of the stream, in nvkv_ring_visible's order), Q_fk is the
 * row with its 44-channel frame segment rotated by f_q - f_k (f_q the RoPE
 * index of the row's own frame) and its h and w segments at the row's (h,
 * w), all in float as nvfp4_kv_append_spatial_rope rotates K; it is
 * quantized with the cache's block rule under the row's global scale s_gq =
 * fl32(p / 2688), p the largest pair magnitude fl32(sqrt(fl32(x^2) +
 * fl32(y^2))) of the row (which no rotation changes; 1 if not a normal
 * float).  Then the dot product of the dequantized Q_fk and cached K' rows
 * equals the rotated q . k of chunk_attention_nvfp4kv up to the two
 * quantizations.  q: device bf16 [B][Lq][H][128], pre-RoPE.  Outputs, device:
 * codes [B][H][Lq][S+W][64] (8-byte aligned), scales [B][H][Lq][S+W][8]
 * (E4M3 codes), s_gq [B][H][Lq] f32; entries j >= the stream's visible
 * frames are not written.  NVKV_ERR_STATE before the first append;
 * NVKV_ERR_UNSUPPORTED unless the RoPE split is 44/42/42 and grid_h + grid_w
 * <= 100. */
NVKV_API nvkv_status nvkv_fp4qk_quantize_q(const nvkv_desc *desc, const nvkv_ring *ring,
                                           const void *q, uint8_t *codes, uint8_t *scales,
                                           float *s_gq, nvkv_stream stream);

/* The contraction of the same reading on the block-scaled tensor cores
 * (tcgen05.mma kind::mxf4nvf4, E2M1 operands, UE4M3 block scales per 16):
 * the logit of every query row against every visible cached key,
 *   out = (sum over blocks of sA sB sum of code products) * s_gq * s_g(K),
 * i.e. the dot product of the dequantized Q_fk and K' rows (without the
 * 1/sqrt(128) of the softmax).  q_codes, q_scales, s_gq: the outputs of
 * nvkv_fp4qk_quantize_q for this step; the cache must have been filled by
 * nvfp4_kv_append_spatial_rope.  out: device f32 [B][H][Lq][S+W][Ts], entry
 * (row, j, i) the logit against token i of the stream's visible frame j
 * (entries of frames past the visible ones are not written).  It writes the
 * whole logit matrix (Lq x visible keys per head), so it suits small shapes;
 * a fused attention would keep each tile in TMEM.  NVKV_ERR_STATE for a bf16
 * cache or before the first append; NVKV_ERR_ALIGNMENT unless q_codes and
 * k_data are 16-byte, the scale arrays 8-byte and s_gq and out 4-byte
 * aligned; the status word receives NVKV_ERR_TIMEOUT if an MMA wait runs
 * out. */
NVKV_API nvkv_status nvkv_fp4qk_scores(const nvkv_desc *desc, const nvkv_cache *cache,
                                       const nvkv_ring *ring, const uint8_t *q_codes,
                                       const uint8_t *q_scales, const float *s_gq, float *out,
                                       nvkv_stream stream);

/* The bf16-KV twin: same slot logic, the chunk's bf16 K/V copied as is. */
NVKV_API nvkv_status bf16_kv_append(const nvkv_desc *desc, const nvkv_cache *cache, nvkv_ring *ring,
                           const void *k, const void *v, nvkv_stream stream);

/* In-place overwrite of the newest chunk, for the denoising steps of one AR
 * step ("NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
 * generation", section "NVFP4, sequence parallel and the async decode path":
 * in-place quantized KV-cache updates; the generator refines each chunk over
 * 2 or 4 denoising steps, and every step recomputes that chunk's K/V).
 * k, v: device bf16 [B][Lq][H][128], the chunk's new K/V.  Quantizes them
 * (NVFP4) or copies them (bf16 twin) into the physical slots of every
 * stream's C newest frames, the same slots their append used; the ring is
 * not modified and eviction does not run.  While the first chunk is the only
 * chunk appended (ring->steps == 1) the overwrite measures that chunk's amax
 * again and fixes s_g from the new values; afterwards s_g stays as it is.
 * NVKV_ERR_STATE if no chunk was appended yet or the desc and ring disagree;
 * the other errors as for the appends. */
NVKV_API nvkv_status nvfp4_kv_overwrite(const nvkv_desc *desc, const nvkv_cache *cache,
                                        const nvkv_ring *ring, const void *k, const void *v,
                                        nvkv_stream stream);
NVKV_API nvkv_status bf16_kv_overwrite(const nvkv_desc *desc, const nvkv_cache *cache,
                                       const nvkv_ring *ring, const void *k, const void *v,
                                       nvkv_stream stream);

/* Device workspace the attention calls need on the current device (0 for an
 * invalid desc or without a device).  The attention kernels run a persistent
 * grid of CTA pairs; query tiles cut between pairs leave partial results
 * here and the last pair to finish merges them.  The caller allocates it once,
 * 16-byte aligned, and zero-fills it before first use; every call leaves it
 * zeroed again.  Calls sharing a workspace must not overlap on the GPU. */
NVKV_API size_t nvkv_attention_workspace_bytes(const nvkv_desc *desc);

/* Block-causal chunk attention of the newest chunk.  q: device bf16
 * [B][Lq][H][128] before RoPE; out: device bf16 [B][Lq][H][128]; lse: NULL or
 * device f32 [B][H][Lq] (natural-log softmax normaliser, max included).
 * Every query of the chunk sees every token of every visible frame (its own
 * chunk included, in full).  Keys are read from the cache, dequantized and
 * rotated by 3D RoPE at (their frame's RoPE index, h, w); queries are rotated
 * at (the RoPE index of their own frame, h, w).  Logits use 1/sqrt(128).
 * Any finite bf16 q is accepted: each query row is multiplied by the power of
 * two 2^e that puts its largest |q| in [2^13, 2^14) before it is rounded to
 * the f16 tensor-core operand, and 2^-e is folded into that row's logit
 * scale, which leaves the logits of rows already inside f16's range
 * unchanged bit for bit.
 * workspace: device memory of nvkv_attention_workspace_bytes() bytes (else
 * NVKV_ERR_CAPACITY).  NVKV_ERR_STATE if nothing was appended yet;
 * NVKV_ERR_UNSUPPORTED for a RoPE
 * split other than 44/42/42, grid_h or grid_w above 256, or RoPE tables too
 * large for one CTA's shared memory: 176 (frames resident) + 168 (grid_h +
 * grid_w) bytes above about 104 KB (only near the largest grids with many
 * frames). */
NVKV_API nvkv_status chunk_attention_nvfp4kv(const nvkv_desc *desc, const nvkv_cache *cache,
                                    const nvkv_ring *ring, const void *q, void *out, float *lse,
                                    void *workspace, size_t workspace_bytes, nvkv_stream stream);

/* The bf16-KV twin of chunk_attention_nvfp4kv.  Both attention calls feed the
 * tensor cores f16 operands with f32 accumulation.  Q is range-scaled per row
 * as in chunk_attention_nvfp4kv; the twin's cached K and V are converted to
 * f16 as they are, so they must lie inside the f16 range (|K| and |V| below
 * 65504 after RoPE), and values below 2^-14 lose precision. */
NVKV_API nvkv_status chunk_attention_bf16kv(const nvkv_desc *desc, const nvkv_cache *cache,
                                   const nvkv_ring *ring, const void *q, void *out, float *lse,
                                   void *workspace, size_t workspace_bytes, nvkv_stream stream);

/* The K/V projection of a chunk, the step before the append, on the tensor
 * cores: K = x W_k^T, V = x W_v^T with bf16 inputs and f32 accumulation,
 * rounded to bf16 (round to nearest even).  x: device bf16 [B][Lq][hidden]
 * (the chunk's hidden states, token-major), w_k, w_v: device bf16
 * [H*128][hidden] (output channel h*128 + d in row h*128 + d), k_out, v_out:
 * device bf16 [B][Lq][H][128].  status: device int32, cleared by the caller,
 * receives NVKV_ERR_TIMEOUT if a pipeline wait runs out.  hidden must be a
 * positive multiple of 64 (else NVKV_ERR_UNSUPPORTED); the desc must be a
 * whole cache (shard_count 1).  All pointers 16-byte aligned. */
NVKV_API nvkv_status nvkv_kv_project(const nvkv_desc *desc, const void *x, int hidden,
                                     const void *w_k, const void *w_v, void *k_out, void *v_out,
                                     int32_t *status, nvkv_stream stream);

/* The projection with the quantize-append fused into its epilogue ("NVlabs/
 * LongLive 2.0: NVFP4 parallel infrastructure for long video generation",
 * section "NVFP4, sequence parallel and the async decode path": in-place
 * quantized KV-cache updates): each token-head row of K and V is rounded to
 * bf16 as nvkv_kv_project would return it and quantized to NVFP4 straight
 * into the ring slot nvfp4_kv_append would give it; the bf16 K/V never
 * reaches memory.  The result is exactly nvkv_kv_project followed by
 * nvfp4_kv_append.  The first append of a cache fixes s_g from the whole
 * chunk's amax, which the epilogue cannot know: it runs nvkv_kv_project into
 * scratch (device, >= 2 * B * Lq * H * 128 * 2 bytes, else NVKV_ERR_CAPACITY)
 * and then nvfp4_kv_append; later appends need no scratch (may be NULL).
 * Ring update and errors as nvfp4_kv_append, and as nvkv_kv_project. */
NVKV_API nvkv_status nvfp4_kv_project_append(const nvkv_desc *desc, const nvkv_cache *cache,
                                             nvkv_ring *ring, const void *x, int hidden,
                                             const void *w_k, const void *w_v, void *scratch,
                                             size_t scratch_bytes, nvkv_stream stream);

/* Merge of the partial attentions of disjoint key sets (the shards of a
 * sequence-parallel KV split) for query rows [q0, q1):
 *   L = log sum_j exp(L_j),  O = sum_j exp(L_j - L) O_j,
 * which is the softmax attention over the union of the key sets (a part
 * whose L_j is -inf, no keys, is skipped).  o_parts, lse_parts: host arrays
 * of n_parts device pointers, part j's out ([B][Lq][H][128] bf16) and lse
 * ([B][H][Lq] f32) of an attention call.  They may point into another GPU's
 * memory mapped into this process (peer access or IPC), so that one kernel
 * does the exchange and the merge: the caller orders this call after every
 * part is written.  out: device bf16 [B][q1-q0][H][128]; lse_out: NULL or
 * device f32 [B][H][q1-q0].  NVKV_ERR_INVALID_ARG for n_parts outside
 * 1..NVKV_MAX_SHARDS, a null pointer or a bad range; NVKV_ERR_ALIGNMENT
 * unless the out pointers are 16-byte and the lse pointers 4-byte aligned. */
NVKV_API nvkv_status nvkv_lse_merge(int n_parts, const void *const *o_parts,
                                    const float *const *lse_parts, int B, int H, int Lq, int q0,
                                    int q1, void *out, float *lse_out, nvkv_stream stream);

/* One step's exchange of a sequence-parallel split: a cross-rank barrier on
 * device flags, bounded in time, fused with nvkv_lse_merge in one kernel, so
 * that no rank reads a peer's part before the peer has finished writing it.
 * This rank is `rank` of n_parts ranks; o_parts, lse_parts and the result as
 * in nvkv_lse_merge.  flags: host array of n_parts device pointers, flags[j]
 * rank j's signal array of NVKV_MAX_SHARDS uint32 (memory this process can
 * store to and load from: a peer mapping or symmetric memory), zero-filled on
 * every rank before any rank's first call.  epoch: 1 on the first call, one
 * more on each later call, the same sequence on every rank (wrap-safe).  Each
 * CTA stores epoch into flags[j][rank] for every j (release, system scope:
 * this rank's part, written by earlier work on `stream`, is visible to a
 * rank that sees the value), then waits until flags[rank][j] has reached
 * epoch for every j.  A wait longer than timeout_us, or a nonzero *status,
 * ends it: the kernel writes NVKV_ERR_TIMEOUT to *status (if it was zero) and
 * skips the merge (the output is undefined); nothing traps or hangs.  A rank
 * reuses its part's memory only after its next call's barrier, by which time
 * every rank has finished reading it.  NVKV_ERR_INVALID_ARG as nvkv_lse_merge
 * and for a null flags entry or status, rank outside [0, n_parts), epoch 0 or
 * timeout_us 0; NVKV_ERR_ALIGNMENT for flags or status not 4-byte aligned. */
NVKV_API nvkv_status nvkv_lse_merge_synced(int n_parts, const void *const *o_parts,
                                           const float *const *lse_parts,
                                           uint32_t *const *flags, int rank, uint32_t epoch,
                                           uint32_t timeout_us, int32_t *status, int B, int H,
                                           int Lq, int q0, int q1, void *out, float *lse_out,
                                           nvkv_stream stream);

/* Test hook of the failure path (no counterpart in the paper).  With fault =
 * NVKV_FAULT_SKIP_FIRST_STAGE the next chunk_attention_* call on this thread
 * runs with its staging producer never filling the first stage, so the waits
 * on it run out after their bound (2 s): the kernel writes NVKV_ERR_TIMEOUT
 * to cache->status, unwinds (waiting for its own copies and MMAs) and
 * returns; nothing traps or hangs.  After a timeout the caller clears the
 * status word and zero-fills the workspace again before reusing them; the
 * output of that call is undefined.  NVKV_FAULT_NONE cancels a pending
 * fault. */
enum { NVKV_FAULT_NONE = 0, NVKV_FAULT_SKIP_FIRST_STAGE = 1 };
NVKV_API nvkv_status nvkv_debug_inject_fault(int fault);

/* Diagnostics: the device conversions the append kernel uses, one value per
 * element.  y, t: device f32 [n]; codes: device u8 [n].
 * nvkv_encode_e2m1: E2M1_RNE_sat(y) with negative zero stored as 0.
 * nvkv_encode_block_scale: E4M3_RNE(min(t, 448)) for t >= 0. */
NVKV_API nvkv_status nvkv_encode_e2m1(const float *y, uint8_t *codes, size_t n, nvkv_stream stream);
NVKV_API nvkv_status nvkv_encode_block_scale(const float *t, uint8_t *codes, size_t n, nvkv_stream stream);

NVKV_API const char *nvkv_status_string(nvkv_status status);

/* NVKV_VERSION of the loaded library. */
NVKV_API uint32_t nvkv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NVKV_H */
