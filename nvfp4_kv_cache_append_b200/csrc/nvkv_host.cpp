// C-ABI host layer: descriptor checks, cache sizing, the sink + rolling-window
// ring, and the launch wrappers.  No device allocation, no host sync.
//
// Ring rules (attention sink and multi-shot sink: "NVlabs/LongLive 2.0: NVFP4
// parallel infrastructure for long video generation", section "NVFP4,
// sequence parallel and the async decode path"; relative RoPE: "NVlabs
// LongLive" (refft.com), Core Analysis block "How do KV-cache relative RoPE
// and TriAttention work together"):
//   * capacity S + W frames, the window holding the current chunk;
//   * the first S frames appended are the sink and stay resident;
//   * eviction removes the oldest resident frames that are not sink and not
//     pinned; a chunk goes into the lowest free physical slots;
//   * logical order is sink first, then by age; the RoPE frame index of a
//     resident frame is its logical index;
//   * multi-shot: a chunk of shot s sees the global sink, every frame of shot
//     s and the last frame of each earlier shot; the first chunk of a shot
//     s > 0 is pinned while that shot runs.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "nvkv_internal.h"

namespace {

using nvkv::AppendLaunch;
using nvkv::AttnLaunch;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvkv_status check_desc(const nvkv_desc *d)
{
    if (!d) return NVKV_ERR_INVALID_ARG;
    if (d->magic != NVKV_MAGIC || d->version != NVKV_VERSION) return NVKV_ERR_STATE;
    if (d->D != NVKV_HEAD_DIM) return NVKV_ERR_UNSUPPORTED;
    if (d->B < 1 || d->H < 1 || d->grid_h < 1 || d->grid_w < 1 || d->C < 1 || d->S < 0 ||
        d->W < 1)
        return NVKV_ERR_INVALID_ARG;
    if (d->B > NVKV_MAX_BATCH || d->H > 64 || d->C > NVKV_MAX_CHUNK || d->C > d->W ||
        d->S + d->W > NVKV_MAX_FRAMES || d->grid_h > 65535 || d->grid_w > 65535)
        return NVKV_ERR_UNSUPPORTED;
    if (d->kv_dtype != NVKV_KV_NVFP4 && d->kv_dtype != NVKV_KV_BF16) return NVKV_ERR_INVALID_ARG;
    if (d->rope_split[0] + d->rope_split[1] + d->rope_split[2] != NVKV_HEAD_DIM ||
        (d->rope_split[0] | d->rope_split[1] | d->rope_split[2]) & 1 || d->rope_split[0] < 0 ||
        d->rope_split[1] < 0 || d->rope_split[2] < 0 || !(d->rope_base > 0.0f))
        return NVKV_ERR_INVALID_ARG;
    const int64_t T = (int64_t)d->grid_h * d->grid_w;
    if (d->shard_count < 1 || d->shard_count > NVKV_MAX_SHARDS || d->shard_rank < 0 ||
        d->shard_rank >= d->shard_count || T % d->shard_count)
        return NVKV_ERR_INVALID_ARG;
    const int64_t R = (T / d->shard_count + 1) / 2 * 2 * (d->S + d->W);
    // 32-bit index arithmetic in the kernels
    if (R * d->B * d->H * 128 >= (int64_t(1) << 31) / 2 ||
        T * d->C * d->B * d->H * 128 >= (int64_t(1) << 31) / 2)
        return NVKV_ERR_UNSUPPORTED;
    return NVKV_OK;
}

nvkv_status check_ring(const nvkv_desc *d, const nvkv_ring *r)
{
    if (!r) return NVKV_ERR_INVALID_ARG;
    if (r->magic != NVKV_MAGIC || r->version != NVKV_VERSION) return NVKV_ERR_STATE;
    if (r->B != d->B || r->capacity != d->S + d->W || r->C != d->C || r->S != d->S)
        return NVKV_ERR_STATE;
    for (int b = 0; b < d->B; ++b)
        if (r->s[b].n_resident < 0 || r->s[b].n_resident > r->capacity) return NVKV_ERR_STATE;
    return NVKV_OK;
}

int64_t rows_per_head(const nvkv_desc *d) { return (int64_t)nvkv::slot_rows(d) * (d->S + d->W); }

bool is_visible(const nvkv_ring_stream &s, int i)
{
    return (s.flags[i] & (NVKV_FRAME_SINK | NVKV_FRAME_SHOT_LAST)) || s.frame_shot[i] == s.shot;
}

// Assigns C free physical slots to every stream; fills a.slot.  Does not
// modify the ring.  Returns false if some stream has no room.
bool plan_slots(const nvkv_desc *d, const nvkv_ring *r, int32_t *slot_out)
{
    const int cap = d->S + d->W;
    for (int b = 0; b < d->B; ++b) {
        const nvkv_ring_stream &s = r->s[b];
        if (s.n_resident + d->C > cap) return false;
        bool used[NVKV_MAX_FRAMES] = {};
        for (int i = 0; i < s.n_resident; ++i) used[s.slot[i]] = true;
        int c = 0;
        for (int p = 0; p < cap && c < d->C; ++p)
            if (!used[p]) slot_out[b * d->C + c++] = p;
        if (c < d->C) return false;
    }
    return true;
}

void commit_append(const nvkv_desc *d, nvkv_ring *r, const int32_t *slot)
{
    for (int b = 0; b < d->B; ++b) {
        nvkv_ring_stream &s = r->s[b];
        for (int c = 0; c < d->C; ++c) {
            const int i = s.n_resident++;
            const int fno = s.n_appended++;
            s.slot[i] = slot[b * d->C + c];
            s.frame[i] = fno;
            s.frame_shot[i] = s.shot;
            s.flags[i] = (fno < d->S ? NVKV_FRAME_SINK : 0u) | (s.pin_next ? NVKV_FRAME_PINNED : 0u);
        }
        s.pin_next = 0;
    }
    r->scales_fixed = 1;
    r->steps += 1;
}

// Physical slots of every stream's newest chunk (frames n_appended - C ..
// n_appended - 1), in frame order.  False if a stream has not appended a
// chunk yet or one of those frames is no longer resident.
bool newest_chunk_slots(const nvkv_desc *d, const nvkv_ring *r, int32_t *slot_out)
{
    for (int b = 0; b < d->B; ++b) {
        const nvkv_ring_stream &s = r->s[b];
        const int f0 = s.n_appended - d->C;
        if (f0 < 0) return false;
        int found = 0;
        for (int i = 0; i < s.n_resident; ++i) {
            const int c = s.frame[i] - f0;
            if (c >= 0 && c < d->C) {
                slot_out[b * d->C + c] = s.slot[i];
                ++found;
            }
        }
        if (found != d->C) return false;
    }
    return true;
}

// Quantize-append into C newly assigned slots, the ring then advanced
// (advance = the ring), or, with advance = null, in-place overwrite of the
// newest chunk: same slots, ring unchanged; while the first chunk is the only
// one appended, its overwrite fixes s_g again from the new values.
// amax_scratch: when not null, the NVFP4 amax scratch to use in place of
// cache->amax (which may then be null).
nvkv_status append_common(const nvkv_desc *desc, const nvkv_cache *cache, const nvkv_ring *ring,
                          nvkv_ring *advance, const void *k, const void *v, cudaStream_t stream,
                          int dtype, uint32_t *amax_scratch = nullptr, bool spatial_rope = false)
{
    const bool overwrite = advance == nullptr;
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (desc->kv_dtype != dtype) return NVKV_ERR_STATE;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (!cache || !k || !v || !cache->k_data || !cache->v_data) return NVKV_ERR_INVALID_ARG;
    uint32_t *amax = amax_scratch ? amax_scratch : cache->amax;
    if (dtype == NVKV_KV_NVFP4 && (!cache->k_scales || !cache->v_scales || !amax || !cache->s_g))
        return NVKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(cache->k_data) || !aligned16(cache->v_data) ||
        (dtype == NVKV_KV_NVFP4 && (!aligned16(cache->k_scales) || !aligned16(cache->v_scales))))
        return NVKV_ERR_ALIGNMENT;

    AppendLaunch a{};
    if (overwrite) {
        if (ring->steps < 1 || !newest_chunk_slots(desc, ring, a.slot)) return NVKV_ERR_STATE;
    } else if (!plan_slots(desc, ring, a.slot)) {
        return NVKV_ERR_CAPACITY;
    }
    a.k = k;
    a.v = v;
    a.k_data = cache->k_data;
    a.v_data = cache->v_data;
    a.k_scales = cache->k_scales;
    a.v_scales = cache->v_scales;
    a.amax = amax;
    a.s_g = cache->s_g;
    a.B = desc->B;
    a.H = desc->H;
    a.T = desc->grid_h * desc->grid_w;
    a.Lq = desc->C * a.T;
    a.Ts = nvkv::shard_tokens(desc);
    a.tok_off = nvkv::shard_first_token(desc);
    a.Tr = nvkv::slot_rows(desc);
    a.R = (int)rows_per_head(desc);
    a.C = desc->C;
    a.first = overwrite ? (ring->steps == 1 ? 1 : 0) : (ring->scales_fixed ? 0 : 1);
    a.grid_w = desc->grid_w;
    cudaError_t e;
    if (spatial_rope) {
        // cos and sin of each spatial pair: the fp64 angle pos * base^(-2i/42),
        // cos and sin in fp64, each rounded once to float
        static thread_local nvkv::SpatialRope r;
        for (int ax = 0; ax < 2; ++ax) {
            const int d = desc->rope_split[1 + ax], n = ax ? desc->grid_w : desc->grid_h;
            float2 *tab = ax ? r.w : r.h;
            for (int pos = 0; pos < n; ++pos)
                for (int i = 0; i < d / 2; ++i) {
                    const double ang = (double)pos * std::pow((double)desc->rope_base, -2.0 * i / (double)d);
                    tab[pos * 21 + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
                }
        }
        e = nvkv::launch_nvfp4_append_rope(a, r, stream);
    } else {
        e = (dtype == NVKV_KV_NVFP4) ? nvkv::launch_nvfp4_append(a, stream)
                                     : nvkv::launch_bf16_append(a, stream);
    }
    if (e != cudaSuccess) return NVKV_ERR_CUDA;
    if (!overwrite) commit_append(desc, advance, a.slot);
    return NVKV_OK;
}

// Persistent schedule of the attention kernel: CTA pairs (slots) and the
// tiles per slot.  Each slot holds at most kMaxSegments work segments, so
// very small items raise the slot count (extra pairs run as later waves).
constexpr int kTileKeys = 128;
// one-shot test hook (nvkv_debug_inject_fault), consumed by the next attention call
thread_local int t_fault = NVKV_FAULT_NONE;
constexpr int kMaxSegments = 94;     // the kernel holds 96; two spare

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int schedule_slots(int dev_slots, int64_t total_tiles, int64_t min_item_tiles)
{
    int64_t n = dev_slots;
    if (min_item_tiles > 0) n = std::max<int64_t>(n, ceil_div(total_tiles, kMaxSegments * min_item_tiles));
    return (int)std::min<int64_t>(n, 1 << 20);
}

int query_pairs(const nvkv_desc *d) { return (int)ceil_div(ceil_div((int64_t)d->C * d->grid_h * d->grid_w, 128), 2); }

nvkv_status attention_common(const nvkv_desc *desc, const nvkv_cache *cache,
                             const nvkv_ring *ring, const void *q, void *out, float *lse,
                             void *ws, size_t ws_bytes, cudaStream_t stream, int dtype)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (desc->kv_dtype != dtype) return NVKV_ERR_STATE;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (ring->steps < 1) return NVKV_ERR_STATE;
    if (!cache || !q || !out || !cache->k_data || !cache->v_data || !cache->status)
        return NVKV_ERR_INVALID_ARG;
    if (dtype == NVKV_KV_NVFP4 && (!cache->k_scales || !cache->v_scales || !cache->s_g))
        return NVKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(cache->k_data) ||
        !aligned16(cache->v_data) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (dtype == NVKV_KV_NVFP4 && (!aligned16(cache->k_scales) || !aligned16(cache->v_scales))))
        return NVKV_ERR_ALIGNMENT;

    AttnLaunch a{};
    a.q = q;
    a.out = out;
    a.lse = lse;
    a.k_data = cache->k_data;
    a.v_data = cache->v_data;
    a.k_scales = cache->k_scales;
    a.v_scales = cache->v_scales;
    a.s_g = cache->s_g;
    a.status = cache->status;
    a.B = desc->B;
    a.H = desc->H;
    a.T = desc->grid_h * desc->grid_w;
    a.Lq = desc->C * a.T;
    a.R = (int)rows_per_head(desc);
    a.grid_w = desc->grid_w;
    a.kv_dtype = dtype;
    a.grid_h = desc->grid_h;
    a.inv_T = 1.0f / (float)a.T;
    a.inv_grid_w = 1.0f / (float)desc->grid_w;
    a.Tk = nvkv::shard_tokens(desc);
    a.tok_off = nvkv::shard_first_token(desc);
    // keys are numbered Tr per frame, the padding row of an odd Tk included
    // (masked), so that every run of rows the kernel copies is 16-byte sized
    a.Tr = nvkv::slot_rows(desc);
    a.inv_Tr = 1.0f / (float)a.Tr;
    // the attention kernels are built for the 44/42/42 split and small grids
    if (desc->rope_split[0] != 44 || desc->rope_split[1] != 42 || desc->rope_split[2] != 42 ||
        desc->grid_h > 256 || desc->grid_w > 256)
        return NVKV_ERR_UNSUPPORTED;
    {
        int p = 0;
        for (int ax = 0; ax < 3; ++ax) {
            const int d = desc->rope_split[ax];
            for (int i = 0; i < d / 2; ++i)
                a.theta[p++] = (float)std::pow((double)desc->rope_base, -2.0 * i / (double)d);
        }
    }
    a.n_fpos = 0;
    for (int b = 0; b < desc->B; ++b) {
        const nvkv_ring_stream &s = ring->s[b];
        if (s.n_resident < desc->C) return NVKV_ERR_STATE;
        int n = 0;
        for (int i = 0; i < s.n_resident; ++i)
            if (is_visible(s, i)) {
                a.vis[b][n].slot = (uint16_t)s.slot[i];
                a.vis[b][n].rope_pos = (uint16_t)i;
                ++n;
            }
        a.n_vis[b] = n;
        a.q_pos0[b] = s.n_resident - desc->C;
        if (s.n_resident > a.n_fpos) a.n_fpos = s.n_resident;
    }
    if (!nvkv::attention_fits(a)) return NVKV_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVKV_ERR_CUDA;
    const int dev_slots = nvkv::attention_slots(dev);
    if (dev_slots < 1) return NVKV_ERR_CUDA;
    a.n_pairs = query_pairs(desc);
    int64_t total = 0, min_tiles = INT64_MAX;
    for (int b = 0; b < desc->B; ++b) {
        const int64_t nkt = ceil_div((int64_t)a.n_vis[b] * a.Tr, kTileKeys);
        total += (int64_t)desc->H * a.n_pairs * nkt;
        min_tiles = std::min(min_tiles, nkt);
    }
    a.n_slots = schedule_slots(dev_slots, total, min_tiles);
    if (!ws || ws_bytes < nvkv::attention_workspace_bytes(a.n_slots)) return NVKV_ERR_CAPACITY;
    if (reinterpret_cast<uintptr_t>(ws) & 15u) return NVKV_ERR_ALIGNMENT;
    a.workspace = ws;
    a.fault = t_fault;
    t_fault = NVKV_FAULT_NONE;
    if (nvkv::launch_chunk_attention(a, stream) != cudaSuccess) return NVKV_ERR_CUDA;
    return NVKV_OK;
}

}  // namespace

nvkv_status nvkv::nvfp4_append_with_scratch(const nvkv_desc *desc, const nvkv_cache *cache,
                                            nvkv_ring *ring, const void *k, const void *v,
                                            cudaStream_t stream, uint32_t *amax_scratch)
{
    return append_common(desc, cache, ring, ring, k, v, stream, NVKV_KV_NVFP4, amax_scratch);
}

extern "C" {

nvkv_status nvkv_desc_init(nvkv_desc *desc, int B, int H, int grid_h, int grid_w, int C, int S,
                           int W, int kv_dtype)
{
    if (!desc) return NVKV_ERR_INVALID_ARG;
    std::memset(desc, 0, sizeof(*desc));
    desc->magic = NVKV_MAGIC;
    desc->version = NVKV_VERSION;
    desc->B = B;
    desc->H = H;
    desc->D = NVKV_HEAD_DIM;
    desc->grid_h = grid_h;
    desc->grid_w = grid_w;
    desc->C = C;
    desc->S = S;
    desc->W = W;
    desc->kv_dtype = kv_dtype;
    desc->rope_base = 10000.0f;
    desc->rope_split[0] = 44;
    desc->rope_split[1] = 42;
    desc->rope_split[2] = 42;
    desc->shard_rank = 0;
    desc->shard_count = 1;
    return check_desc(desc);
}

nvkv_status nvkv_desc_set_shard(nvkv_desc *desc, int rank, int count)
{
    if (!desc) return NVKV_ERR_INVALID_ARG;
    nvkv_desc d = *desc;
    d.shard_rank = rank;
    d.shard_count = count;
    nvkv_status st = check_desc(&d);
    if (st != NVKV_OK) return st;
    *desc = d;
    return NVKV_OK;
}

size_t nvkv_plane_bytes(const nvkv_desc *d, int plane)
{
    if (check_desc(d) != NVKV_OK) return 0;
    const size_t rows = (size_t)rows_per_head(d) * d->B * d->H;
    const bool fp4 = d->kv_dtype == NVKV_KV_NVFP4;
    switch (plane) {
    case NVKV_PLANE_K_DATA:
    case NVKV_PLANE_V_DATA: return rows * (fp4 ? 64 : 256);
    // +16 bytes: scale runs are copied in 16-byte granules that may reach one
    // row past the last one
    case NVKV_PLANE_K_SCALES:
    case NVKV_PLANE_V_SCALES: return fp4 ? rows * 8 + 16 : 0;
    case NVKV_PLANE_AMAX: return fp4 ? sizeof(uint32_t) * 2 * d->B * d->H : 0;
    case NVKV_PLANE_SCALE_G: return fp4 ? sizeof(float) * 2 * d->B * d->H : 0;
    case NVKV_PLANE_STATUS: return sizeof(int32_t);
    default: return 0;
    }
}

nvkv_status nvkv_ring_init(const nvkv_desc *desc, nvkv_ring *ring)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (!ring) return NVKV_ERR_INVALID_ARG;
    std::memset(ring, 0, sizeof(*ring));
    ring->magic = NVKV_MAGIC;
    ring->version = NVKV_VERSION;
    ring->B = desc->B;
    ring->capacity = desc->S + desc->W;
    ring->C = desc->C;
    ring->S = desc->S;
    return NVKV_OK;
}

nvkv_status kv_ring_evict(const nvkv_desc *desc, nvkv_ring *ring, int n_frames)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (n_frames < 0) return NVKV_ERR_INVALID_ARG;
    for (int b = 0; b < desc->B; ++b) {
        const nvkv_ring_stream &s = ring->s[b];
        int n = 0;
        for (int i = 0; i < s.n_resident; ++i)
            if (!(s.flags[i] & (NVKV_FRAME_SINK | NVKV_FRAME_PINNED))) ++n;
        if (n < n_frames) return NVKV_ERR_CAPACITY;
    }
    for (int b = 0; b < desc->B; ++b) {
        nvkv_ring_stream &s = ring->s[b];
        int dropped = 0, w = 0;
        for (int i = 0; i < s.n_resident; ++i) {
            const bool evictable = !(s.flags[i] & (NVKV_FRAME_SINK | NVKV_FRAME_PINNED));
            if (evictable && dropped < n_frames) {
                ++dropped;
                continue;
            }
            s.slot[w] = s.slot[i];
            s.frame[w] = s.frame[i];
            s.frame_shot[w] = s.frame_shot[i];
            s.flags[w] = s.flags[i];
            ++w;
        }
        s.n_resident = w;
    }
    return NVKV_OK;
}

nvkv_status kv_ring_begin_shot(const nvkv_desc *desc, nvkv_ring *ring, int b, int shot_id)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (b < 0 || b >= desc->B) return NVKV_ERR_INVALID_ARG;
    nvkv_ring_stream &s = ring->s[b];
    if (shot_id < s.shot) return NVKV_ERR_INVALID_ARG;
    if (shot_id == s.shot) return NVKV_OK;
    if (s.n_resident > 0) s.flags[s.n_resident - 1] |= NVKV_FRAME_SHOT_LAST;
    for (int i = 0; i < s.n_resident; ++i) s.flags[i] &= ~NVKV_FRAME_PINNED;
    s.shot = shot_id;
    s.pin_next = shot_id > 0 ? 1 : 0;
    return NVKV_OK;
}

int nvkv_ring_visible(const nvkv_desc *desc, const nvkv_ring *ring, int b, int32_t *slots,
                      int32_t *rope_pos, int32_t *frames, int32_t *query_pos0)
{
    if (check_desc(desc) != NVKV_OK || check_ring(desc, ring) != NVKV_OK || b < 0 || b >= desc->B)
        return -1;
    const nvkv_ring_stream &s = ring->s[b];
    int n = 0;
    for (int i = 0; i < s.n_resident; ++i)
        if (is_visible(s, i)) {
            if (slots) slots[n] = s.slot[i];
            if (rope_pos) rope_pos[n] = i;
            if (frames) frames[n] = s.frame[i];
            ++n;
        }
    if (query_pos0) *query_pos0 = s.n_resident - desc->C;
    return n;
}

nvkv_status nvkv_ring_push_chunk(const nvkv_desc *desc, nvkv_ring *ring, int32_t *slots_out)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    int32_t slot[NVKV_MAX_BATCH * NVKV_MAX_CHUNK];
    if (!plan_slots(desc, ring, slot)) return NVKV_ERR_CAPACITY;
    commit_append(desc, ring, slot);
    if (slots_out) std::memcpy(slots_out, slot, sizeof(int32_t) * desc->B * desc->C);
    return NVKV_OK;
}

nvkv_status nvfp4_kv_append(const nvkv_desc *desc, const nvkv_cache *cache, nvkv_ring *ring,
                            const void *k, const void *v, nvkv_stream stream)
{
    return append_common(desc, cache, ring, ring, k, v, (cudaStream_t)stream, NVKV_KV_NVFP4);
}

nvkv_status bf16_kv_append(const nvkv_desc *desc, const nvkv_cache *cache, nvkv_ring *ring,
                           const void *k, const void *v, nvkv_stream stream)
{
    return append_common(desc, cache, ring, ring, k, v, (cudaStream_t)stream, NVKV_KV_BF16);
}

nvkv_status nvfp4_kv_append_spatial_rope(const nvkv_desc *desc, const nvkv_cache *cache,
                                         nvkv_ring *ring, const void *k, const void *v,
                                         nvkv_stream stream)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (desc->rope_split[0] != 44 || desc->rope_split[1] != 42 || desc->rope_split[2] != 42 ||
        desc->grid_h > nvkv::kRopeAppendMaxGrid || desc->grid_w > nvkv::kRopeAppendMaxGrid)
        return NVKV_ERR_UNSUPPORTED;
    return append_common(desc, cache, ring, ring, k, v, (cudaStream_t)stream, NVKV_KV_NVFP4,
                         nullptr, true);
}

nvkv_status nvkv_fp4qk_quantize_q(const nvkv_desc *desc, const nvkv_ring *ring, const void *q,
                                  uint8_t *codes, uint8_t *scales, float *s_gq,
                                  nvkv_stream stream)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (ring->steps < 1) return NVKV_ERR_STATE;
    if (!q || !codes || !scales || !s_gq) return NVKV_ERR_INVALID_ARG;
    if (!aligned16(q) || (reinterpret_cast<uintptr_t>(codes) & 7u) ||
        (reinterpret_cast<uintptr_t>(s_gq) & 3u))
        return NVKV_ERR_ALIGNMENT;
    if (desc->rope_split[0] != 44 || desc->rope_split[1] != 42 || desc->rope_split[2] != 42 ||
        desc->grid_h + desc->grid_w > nvkv::kQfkMaxSpatial)
        return NVKV_ERR_UNSUPPORTED;
    static thread_local nvkv::QfkLaunch a;
    a = nvkv::QfkLaunch{};
    a.q = q;
    a.codes = codes;
    a.scales = scales;
    a.s_gq = s_gq;
    a.B = desc->B;
    a.H = desc->H;
    a.T = desc->grid_h * desc->grid_w;
    a.Lq = desc->C * a.T;
    a.grid_h = desc->grid_h;
    a.grid_w = desc->grid_w;
    a.max_vis = desc->S + desc->W;
    for (int b = 0; b < desc->B; ++b) {
        const nvkv_ring_stream &s = ring->s[b];
        if (s.n_resident < desc->C) return NVKV_ERR_STATE;
        int n = 0;
        for (int i = 0; i < s.n_resident; ++i)
            if (is_visible(s, i)) a.vis_pos[b][n++] = (uint8_t)i;
        a.n_vis[b] = n;
        a.q_pos0[b] = s.n_resident - desc->C;
    }
    // cos and sin of the fp64 angle pos * base^(-2i/d), each rounded once to float
    auto cs = [&](int pos, int i, int d) {
        const double ang = (double)pos * std::pow((double)desc->rope_base, -2.0 * i / (double)d);
        return make_float2((float)std::cos(ang), (float)std::sin(ang));
    };
    for (int dpos = -(nvkv::kQfkMaxChunk - 1); dpos < NVKV_MAX_FRAMES; ++dpos)
        for (int i = 0; i < 22; ++i)
            a.fr[(dpos + nvkv::kQfkMaxChunk - 1) * 22 + i] = cs(dpos, i, desc->rope_split[0]);
    for (int pos = 0; pos < desc->grid_h; ++pos)
        for (int i = 0; i < 21; ++i) a.sp[pos * 21 + i] = cs(pos, i, desc->rope_split[1]);
    for (int pos = 0; pos < desc->grid_w; ++pos)
        for (int i = 0; i < 21; ++i)
            a.sp[(desc->grid_h + pos) * 21 + i] = cs(pos, i, desc->rope_split[2]);
    return nvkv::launch_fp4qk_quantize_q(a, (cudaStream_t)stream) == cudaSuccess ? NVKV_OK
                                                                                : NVKV_ERR_CUDA;
}

nvkv_status nvkv_fp4qk_scores(const nvkv_desc *desc, const nvkv_cache *cache,
                              const nvkv_ring *ring, const uint8_t *q_codes,
                              const uint8_t *q_scales, const float *s_gq, float *out,
                              nvkv_stream stream)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (desc->kv_dtype != NVKV_KV_NVFP4) return NVKV_ERR_STATE;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (ring->steps < 1) return NVKV_ERR_STATE;
    if (!cache || !cache->k_data || !cache->k_scales || !cache->s_g || !cache->status || !q_codes ||
        !q_scales || !s_gq || !out)
        return NVKV_ERR_INVALID_ARG;
    if (!aligned16(q_codes) || (reinterpret_cast<uintptr_t>(q_scales) & 7u) ||
        !aligned16(cache->k_data) || (reinterpret_cast<uintptr_t>(cache->k_scales) & 7u) ||
        (reinterpret_cast<uintptr_t>(s_gq) & 3u) || (reinterpret_cast<uintptr_t>(out) & 3u))
        return NVKV_ERR_ALIGNMENT;
    nvkv::ScoreLaunch a{};
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.s_gq = s_gq;
    a.k_codes = static_cast<const uint8_t *>(cache->k_data);
    a.k_scales = static_cast<const uint8_t *>(cache->k_scales);
    a.s_gk = cache->s_g;
    a.out = out;
    a.status = cache->status;
    a.B = desc->B;
    a.H = desc->H;
    a.Lq = desc->C * desc->grid_h * desc->grid_w;
    a.R = (int)rows_per_head(desc);
    a.Tk = nvkv::shard_tokens(desc);
    a.Tr = nvkv::slot_rows(desc);
    a.max_vis = desc->S + desc->W;
    for (int b = 0; b < desc->B; ++b) {
        const nvkv_ring_stream &s = ring->s[b];
        int n = 0;
        for (int i = 0; i < s.n_resident; ++i)
            if (is_visible(s, i)) a.vis_slot[b][n++] = (uint16_t)s.slot[i];
        a.n_vis[b] = n;
    }
    return nvkv::launch_fp4qk_scores(a, (cudaStream_t)stream) == cudaSuccess ? NVKV_OK : NVKV_ERR_CUDA;
}

nvkv_status nvfp4_kv_overwrite(const nvkv_desc *desc, const nvkv_cache *cache,
                               const nvkv_ring *ring, const void *k, const void *v,
                               nvkv_stream stream)
{
    return append_common(desc, cache, ring, nullptr, k, v, (cudaStream_t)stream, NVKV_KV_NVFP4);
}

nvkv_status bf16_kv_overwrite(const nvkv_desc *desc, const nvkv_cache *cache,
                              const nvkv_ring *ring, const void *k, const void *v,
                              nvkv_stream stream)
{
    return append_common(desc, cache, ring, nullptr, k, v, (cudaStream_t)stream, NVKV_KV_BF16);
}

size_t nvkv_attention_workspace_bytes(const nvkv_desc *desc)
{
    if (check_desc(desc) != NVKV_OK) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const int dev_slots = nvkv::attention_slots(dev);
    if (dev_slots < 1) return 0;
    // bound over every ring state: at most S + W visible frames, at least the
    // chunk's own C frames (keys are numbered slot_rows per frame)
    const int64_t T = nvkv::slot_rows(desc);
    const int64_t max_tiles = ceil_div((desc->S + desc->W) * T, kTileKeys);
    const int64_t min_tiles = ceil_div(desc->C * T, kTileKeys);
    const int64_t total = (int64_t)desc->B * desc->H * query_pairs(desc) * max_tiles;
    return nvkv::attention_workspace_bytes(schedule_slots(dev_slots, total, min_tiles));
}

nvkv_status chunk_attention_nvfp4kv(const nvkv_desc *desc, const nvkv_cache *cache,
                                    const nvkv_ring *ring, const void *q, void *out, float *lse,
                                    void *workspace, size_t workspace_bytes, nvkv_stream stream)
{
    return attention_common(desc, cache, ring, q, out, lse, workspace, workspace_bytes,
                            (cudaStream_t)stream, NVKV_KV_NVFP4);
}

nvkv_status chunk_attention_bf16kv(const nvkv_desc *desc, const nvkv_cache *cache,
                                   const nvkv_ring *ring, const void *q, void *out, float *lse,
                                   void *workspace, size_t workspace_bytes, nvkv_stream stream)
{
    return attention_common(desc, cache, ring, q, out, lse, workspace, workspace_bytes,
                            (cudaStream_t)stream, NVKV_KV_BF16);
}

namespace {

nvkv_status check_project(const nvkv_desc *desc, const void *x, int hidden, const void *w_k,
                          const void *w_v)
{
    nvkv_status st = check_desc(desc);
    if (st != NVKV_OK) return st;
    if (!x || !w_k || !w_v) return NVKV_ERR_INVALID_ARG;
    if (hidden < 64 || hidden % 64) return NVKV_ERR_UNSUPPORTED;
    if (desc->shard_count != 1) return NVKV_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w_k) || !aligned16(w_v)) return NVKV_ERR_ALIGNMENT;
    return NVKV_OK;
}

nvkv::ProjLaunch project_launch(const nvkv_desc *desc, int hidden)
{
    nvkv::ProjLaunch p{};
    p.T = desc->grid_h * desc->grid_w;
    p.Lq = desc->C * p.T;
    p.B = desc->B;
    p.H = desc->H;
    p.C = desc->C;
    p.M = desc->B * p.Lq;
    p.hidden = hidden;
    p.R = (int)rows_per_head(desc);
    p.Tr = nvkv::slot_rows(desc);
    return p;
}

}  // namespace

nvkv_status nvkv_kv_project(const nvkv_desc *desc, const void *x, int hidden, const void *w_k,
                            const void *w_v, void *k_out, void *v_out, int32_t *status,
                            nvkv_stream stream)
{
    nvkv_status st = check_project(desc, x, hidden, w_k, w_v);
    if (st != NVKV_OK) return st;
    if (!k_out || !v_out || !status) return NVKV_ERR_INVALID_ARG;
    if (!aligned16(k_out) || !aligned16(v_out)) return NVKV_ERR_ALIGNMENT;
    nvkv::ProjLaunch p = project_launch(desc, hidden);
    p.mode = 0;
    p.k_out = k_out;
    p.v_out = v_out;
    p.status = status;
    return nvkv::launch_kv_project(p, x, w_k, w_v, (cudaStream_t)stream) == cudaSuccess
               ? NVKV_OK
               : NVKV_ERR_CUDA;
}

nvkv_status nvfp4_kv_project_append(const nvkv_desc *desc, const nvkv_cache *cache,
                                    nvkv_ring *ring, const void *x, int hidden, const void *w_k,
                                    const void *w_v, void *scratch, size_t scratch_bytes,
                                    nvkv_stream stream)
{
    nvkv_status st = check_project(desc, x, hidden, w_k, w_v);
    if (st != NVKV_OK) return st;
    if (desc->kv_dtype != NVKV_KV_NVFP4) return NVKV_ERR_STATE;
    if ((st = check_ring(desc, ring)) != NVKV_OK) return st;
    if (!cache || !cache->k_data || !cache->v_data || !cache->k_scales || !cache->v_scales ||
        !cache->amax || !cache->s_g || !cache->status)
        return NVKV_ERR_INVALID_ARG;
    if (!aligned16(cache->k_data) || !aligned16(cache->v_data) || !aligned16(cache->k_scales) ||
        !aligned16(cache->v_scales))
        return NVKV_ERR_ALIGNMENT;
    nvkv::ProjLaunch p = project_launch(desc, hidden);
    p.status = cache->status;
    if (!ring->scales_fixed) {
        // first chunk: s_g comes from the whole chunk's amax, so the
        // projection goes to bf16 first and the regular append follows
        const size_t one = (size_t)p.M * p.H * 128 * 2;
        if (!scratch || scratch_bytes < 2 * one) return NVKV_ERR_CAPACITY;
        if (!aligned16(scratch)) return NVKV_ERR_ALIGNMENT;
        {
            int32_t slot[NVKV_MAX_BATCH * NVKV_MAX_CHUNK];
            if (!plan_slots(desc, ring, slot)) return NVKV_ERR_CAPACITY;
        }
        p.mode = 0;
        p.k_out = scratch;
        p.v_out = static_cast<uint8_t *>(scratch) + one;
        if (nvkv::launch_kv_project(p, x, w_k, w_v, (cudaStream_t)stream) != cudaSuccess)
            return NVKV_ERR_CUDA;
        return append_common(desc, cache, ring, ring, p.k_out, p.v_out, (cudaStream_t)stream,
                             NVKV_KV_NVFP4);
    }
    if (!plan_slots(desc, ring, p.slot)) return NVKV_ERR_CAPACITY;
    p.mode = 1;
    p.k_data = cache->k_data;
    p.v_data = cache->v_data;
    p.k_scales = cache->k_scales;
    p.v_scales = cache->v_scales;
    p.s_g = cache->s_g;
    if (nvkv::launch_kv_project(p, x, w_k, w_v, (cudaStream_t)stream) != cudaSuccess)
        return NVKV_ERR_CUDA;
    commit_append(desc, ring, p.slot);
    return NVKV_OK;
}

namespace {

nvkv_status merge_setup(int n_parts, const void *const *o_parts, const float *const *lse_parts,
                        int B, int H, int Lq, int q0, int q1, void *out, float *lse_out,
                        nvkv::MergeLaunch &m)
{
    if (n_parts < 1 || n_parts > NVKV_MAX_SHARDS || !o_parts || !lse_parts || !out || B < 1 ||
        H < 1 || Lq < 1 || q0 < 0 || q1 > Lq || q0 >= q1)
        return NVKV_ERR_INVALID_ARG;
    if ((int64_t)B * Lq * H * 128 >= (int64_t(1) << 31)) return NVKV_ERR_UNSUPPORTED;
    m = nvkv::MergeLaunch{};
    for (int j = 0; j < n_parts; ++j) {
        if (!o_parts[j] || !lse_parts[j]) return NVKV_ERR_INVALID_ARG;
        if (!aligned16(o_parts[j]) || (reinterpret_cast<uintptr_t>(lse_parts[j]) & 3u))
            return NVKV_ERR_ALIGNMENT;
        m.o[j] = o_parts[j];
        m.lse[j] = lse_parts[j];
    }
    if (!aligned16(out) || (reinterpret_cast<uintptr_t>(lse_out) & 3u)) return NVKV_ERR_ALIGNMENT;
    m.n = n_parts;
    m.B = B;
    m.H = H;
    m.Lq = Lq;
    m.q0 = q0;
    m.nq = q1 - q0;
    m.out = out;
    m.lse_out = lse_out;
    return NVKV_OK;
}

}  // namespace

nvkv_status nvkv_lse_merge(int n_parts, const void *const *o_parts, const float *const *lse_parts,
                           int B, int H, int Lq, int q0, int q1, void *out, float *lse_out,
                           nvkv_stream stream)
{
    nvkv::MergeLaunch m;
    const nvkv_status st = merge_setup(n_parts, o_parts, lse_parts, B, H, Lq, q0, q1, out, lse_out, m);
    if (st != NVKV_OK) return st;
    return nvkv::launch_lse_merge(m, (cudaStream_t)stream) == cudaSuccess ? NVKV_OK : NVKV_ERR_CUDA;
}

nvkv_status nvkv_lse_merge_synced(int n_parts, const void *const *o_parts,
                                  const float *const *lse_parts, uint32_t *const *flags, int rank,
                                  uint32_t epoch, uint32_t timeout_us, int32_t *status, int B,
                                  int H, int Lq, int q0, int q1, void *out, float *lse_out,
                                  nvkv_stream stream)
{
    nvkv::MergeLaunch m;
    const nvkv_status st = merge_setup(n_parts, o_parts, lse_parts, B, H, Lq, q0, q1, out, lse_out, m);
    if (st != NVKV_OK) return st;
    if (!flags || !status || rank < 0 || rank >= n_parts || epoch == 0 || timeout_us == 0)
        return NVKV_ERR_INVALID_ARG;
    for (int j = 0; j < n_parts; ++j) {
        if (!flags[j]) return NVKV_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(flags[j]) & 3u) return NVKV_ERR_ALIGNMENT;
        m.flags[j] = flags[j];
    }
    if (reinterpret_cast<uintptr_t>(status) & 3u) return NVKV_ERR_ALIGNMENT;
    m.sync = 1;
    m.rank = rank;
    m.epoch = epoch;
    m.timeout_ns = (uint64_t)timeout_us * 1000u;
    m.status = status;
    return nvkv::launch_lse_merge(m, (cudaStream_t)stream) == cudaSuccess ? NVKV_OK : NVKV_ERR_CUDA;
}

nvkv_status nvkv_debug_inject_fault(int fault)
{
    if (fault != NVKV_FAULT_NONE && fault != NVKV_FAULT_SKIP_FIRST_STAGE)
        return NVKV_ERR_INVALID_ARG;
    t_fault = fault;
    return NVKV_OK;
}

nvkv_status nvkv_encode_e2m1(const float *y, uint8_t *codes, size_t n, nvkv_stream stream)
{
    if (n == 0) return NVKV_OK;
    if (!y || !codes) return NVKV_ERR_INVALID_ARG;
    if (n > (size_t(1) << 31)) return NVKV_ERR_UNSUPPORTED;
    return nvkv::launch_encode_e2m1(y, codes, n, (cudaStream_t)stream) == cudaSuccess
               ? NVKV_OK
               : NVKV_ERR_CUDA;
}

nvkv_status nvkv_encode_block_scale(const float *t, uint8_t *codes, size_t n, nvkv_stream stream)
{
    if (n == 0) return NVKV_OK;
    if (!t || !codes) return NVKV_ERR_INVALID_ARG;
    if (n > (size_t(1) << 31)) return NVKV_ERR_UNSUPPORTED;
    return nvkv::launch_encode_block_scale(t, codes, n, (cudaStream_t)stream) == cudaSuccess
               ? NVKV_OK
               : NVKV_ERR_CUDA;
}

const char *nvkv_status_string(nvkv_status s)
{
    switch (s) {
    case NVKV_OK: return "ok";
    case NVKV_ERR_INVALID_ARG: return "invalid argument";
    case NVKV_ERR_UNSUPPORTED: return "unsupported shape or device";
    case NVKV_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case NVKV_ERR_CAPACITY: return "no room in the ring (evict first) or too few evictable frames";
    case NVKV_ERR_STATE: return "descriptor/ring/cache state mismatch";
    case NVKV_ERR_CUDA: return "CUDA launch failed";
    case NVKV_ERR_TIMEOUT: return "device pipeline wait exceeded its bound";
    }
    return "unknown status";
}

uint32_t nvkv_version(void) { return NVKV_VERSION; }

}  // extern "C"
