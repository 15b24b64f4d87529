// Internal launch interface between the C-ABI host layer (nvkv_host.cpp) and
// the CUDA kernels (append.cu, attention.cu).  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvkv.h"

namespace nvkv {

// Quantize-append / bf16 append of one chunk into physical frame slots.
struct AppendLaunch {
    const void *k, *v;               // bf16 [B][Lq][H][128]
    void *k_data, *v_data;           // NVFP4 codes [B][H][R][64] or bf16 [B][H][R][128]
    void *k_scales, *v_scales;       // E4M3 [B][H][R][8] (NVFP4 only)
    uint32_t *amax;                  // [2][B][H]
    float *s_g;                      // [2][B][H]
    int B, H, T, Lq, R, C;           // T tokens per frame, Lq = C * T rows of k, v
    int Ts, tok_off;                 // this shard's tokens of a frame: [tok_off, tok_off + Ts)
    int Tr;                          // rows per frame slot (Ts rounded up to even)
    float inv_Ts;                    // 1/Ts, set by the launchers (frame index by reciprocal)
    int first;                       // 1: measure amax and fix s_g
    int grid_w;                      // tokens per latent row (spatial RoPE variant)
    int32_t slot[NVKV_MAX_BATCH * NVKV_MAX_CHUNK];  // [b * C + c] -> physical slot
};

// cos and sin (float) of the spatial RoPE pairs, for the append that rotates
// K before quantizing it: h[pos * 21 + i] for pair i of the 42-channel h
// segment at row pos, w[pos * 21 + i] likewise for the w segment.  Passed as
// a kernel parameter (30 KB), which bounds the grid.
constexpr int kRopeAppendMaxGrid = 90;
struct SpatialRope {
    float2 h[kRopeAppendMaxGrid * 21];
    float2 w[kRopeAppendMaxGrid * 21];
};
cudaError_t launch_nvfp4_append_rope(const AppendLaunch &a, const SpatialRope &r, cudaStream_t s);

// Q of the block-scaled FP4 Q K^T reading, quantized per visible key frame.
// fr[(dpos + kQfkMaxChunk - 1) * 22 + i]: cos and sin (float) of frame pair i
// at relative index dpos in [-(kQfkMaxChunk - 1), NVKV_MAX_FRAMES - 1];
// sp[pos * 21 + i] for h rows pos < grid_h, sp[(grid_h + pos) * 21 + i] for w
// columns.  Kernel parameter, about 30 KB.
constexpr int kQfkMaxChunk = NVKV_MAX_CHUNK;
constexpr int kQfkMaxSpatial = 100;          // grid_h + grid_w
struct QfkLaunch {
    const void *q;                           // bf16 [B][Lq][H][128]
    uint8_t *codes, *scales;                 // [B][H][Lq][max_vis][64], [..][8]
    float *s_gq;                             // [B][H][Lq]
    int B, H, Lq, T, grid_h, grid_w, max_vis;
    int n_vis[NVKV_MAX_BATCH];
    int q_pos0[NVKV_MAX_BATCH];
    uint8_t vis_pos[NVKV_MAX_BATCH][NVKV_MAX_FRAMES];   // RoPE frame index of visible frame j
    float2 fr[(kQfkMaxChunk - 1 + NVKV_MAX_FRAMES) * 22];
    float2 sp[kQfkMaxSpatial * 21];
};
static_assert(sizeof(QfkLaunch) <= 32764, "kernel parameter space");

// The FP4 contraction of the same reading: logits of every query row against
// every visible key, from the quantized Q_fk (nvkv_fp4qk_quantize_q) and the
// cached K' (nvfp4_kv_append_spatial_rope), on block-scaled tensor-core MMAs.
struct ScoreLaunch {
    const uint8_t *q_codes, *q_scales;      // [B][H][Lq][max_vis][64], [..][8]
    const float *s_gq;                      // [B][H][Lq]
    const uint8_t *k_codes, *k_scales;      // cache planes [B][H][R][64], [..][8]
    const float *s_gk;                      // [B][H] (K's global scales)
    float *out;                             // [B][H][Lq][max_vis][Tk]
    int32_t *status;
    int B, H, Lq, R, Tk, Tr, max_vis;
    int n_vis[NVKV_MAX_BATCH];
    uint16_t vis_slot[NVKV_MAX_BATCH][NVKV_MAX_FRAMES];
};
cudaError_t launch_fp4qk_scores(const ScoreLaunch &a, cudaStream_t s);
cudaError_t launch_fp4qk_quantize_q(const QfkLaunch &a, cudaStream_t s);

// Tokens per frame of the cache a desc describes (the shard's share of each
// frame) and the index of its first token within the frame.
inline int shard_tokens(const nvkv_desc *d)
{
    return d->grid_h * d->grid_w / (d->shard_count > 0 ? d->shard_count : 1);
}
inline int shard_first_token(const nvkv_desc *d) { return d->shard_rank * shard_tokens(d); }
// Rows of a frame slot: the shard's tokens, plus one padding row when their
// count is odd, so that every slot starts on a 16-byte boundary of the
// 8-byte-per-row scale planes.
inline int slot_rows(const nvkv_desc *d) { return (shard_tokens(d) + 1) & ~1; }

cudaError_t launch_nvfp4_append(const AppendLaunch &a, cudaStream_t s);
// nvfp4_kv_append with its amax scratch given by the caller (amax_scratch
// replaces cache->amax, which may be null): the same checks, slots, launch
// and ring update.
nvkv_status nvfp4_append_with_scratch(const nvkv_desc *desc, const nvkv_cache *cache,
                                      nvkv_ring *ring, const void *k, const void *v,
                                      cudaStream_t stream, uint32_t *amax_scratch);
cudaError_t launch_bf16_append(const AppendLaunch &a, cudaStream_t s);
cudaError_t launch_encode_e2m1(const float *y, uint8_t *codes, size_t n, cudaStream_t s);
cudaError_t launch_encode_block_scale(const float *t, uint8_t *codes, size_t n, cudaStream_t s);

// One visible frame of a stream: physical slot and RoPE frame index.
struct VisFrame {
    uint16_t slot;
    uint16_t rope_pos;
};

// Chunk attention over the visible frames of every stream.
struct AttnLaunch {
    const void *q;                   // bf16 [B][Lq][H][128]
    void *out;                       // bf16 [B][Lq][H][128]
    float *lse;                      // f32 [B][H][Lq] or null
    const void *k_data, *v_data;
    const void *k_scales, *v_scales;
    const float *s_g;                // [2][B][H] (NVFP4 only)
    int32_t *status;
    int B, H, T, Lq, R, grid_w;
    int kv_dtype;
    int n_vis[NVKV_MAX_BATCH];       // visible frames per stream
    int q_pos0[NVKV_MAX_BATCH];      // RoPE frame index of the chunk's first frame
    VisFrame vis[NVKV_MAX_BATCH][NVKV_MAX_FRAMES];
    int grid_h;
    float inv_T, inv_grid_w;         // 1/T and 1/grid_w (division by reciprocal + fix-up)
    int Tk, tok_off;                 // cached tokens per frame (the shard's), first one's index
    int Tr;                          // rows per frame slot: Tk, or Tk + 1 (one padding row)
    float inv_Tr;                    // 1/Tr
    int n_fpos;                      // frame positions used: 0 .. n_fpos-1
    float theta[64];                 // RoPE angle per unit position of each channel pair
    void *workspace;                 // split-item partials + counters (zero on first use)
    int n_slots;                     // CTA pairs of the persistent schedule
    int n_pairs;                     // 256-row query tile pairs per (b, h)
    int fault;                       // NVKV_FAULT_* test hook, 0 in normal use
};

// Workspace of the chunk attention for a schedule of n_slots CTA pairs:
// per slot two partial records of 2 x 128 rows x (128 + 2) f32, then counters.
size_t attention_workspace_bytes(int n_slots);
int attention_slots(int device);     // CTA pairs that can be resident at once

cudaError_t launch_chunk_attention(const AttnLaunch &a, cudaStream_t s);
// whether the kernel's shared memory (with the launch's RoPE tables) fits a CTA
bool attention_fits(const AttnLaunch &a);

// K/V projection of one chunk (x [M][hidden] times W^T, W [H*128][hidden],
// bf16 in, f32 accumulate), its epilogue writing bf16 K/V (mode 0) or the
// NVFP4 quantize-append into the ring (mode 1).
struct ProjLaunch {
    int M, hidden;                   // rows of x (B * Lq), hidden (multiple of 64)
    int B, H, Lq, T, R, C;
    int Tr;                          // rows per frame slot
    int mode;
    void *k_out, *v_out;             // mode 0: bf16 [B][Lq][H][128]
    void *k_data, *v_data;           // mode 1: NVFP4 planes of the cache
    void *k_scales, *v_scales;
    const float *s_g;                // [2][B][H]
    int32_t *status;
    int n_pairs;                     // CTA pairs of the persistent grid
    int32_t slot[NVKV_MAX_BATCH * NVKV_MAX_CHUNK];  // mode 1: [b * C + c] -> physical slot
};

cudaError_t launch_kv_project(const ProjLaunch &p, const void *x, const void *w_k, const void *w_v,
                              cudaStream_t s);

// LSE-weighted merge of the partial attentions of disjoint key sets.
struct MergeLaunch {
    const void *o[NVKV_MAX_SHARDS];     // bf16 [B][Lq][H][128] per part
    const float *lse[NVKV_MAX_SHARDS];  // f32 [B][H][Lq] per part
    int n, B, H, Lq, q0, nq;
    void *out;                          // bf16 [B][nq][H][128]
    float *lse_out;                     // f32 [B][H][nq] or null
    // cross-rank barrier fused in front of the merge (sync = 1): rank `rank`
    // stores `epoch` into flags[j][rank] of every part j, then waits until
    // flags[rank][j] reaches epoch for every j, at most timeout_ns
    int sync, rank;
    uint32_t epoch;
    uint32_t *flags[NVKV_MAX_SHARDS];
    uint64_t timeout_ns;
    int32_t *status;
};

cudaError_t launch_lse_merge(const MergeLaunch &m, cudaStream_t s);

}  // namespace nvkv
