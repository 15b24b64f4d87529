// Block-causal chunk attention over the NVFP4 (or bf16) KV ring, sm_100a.
//
// What it computes, per (batch b, head h): the C*T query tokens of the newest
// chunk attend over every token of every visible frame of the ring (the
// chunk's own frames included, in full), softmax(q_rot . k_rot / sqrt(128)) v.
// Keys are cached before RoPE and rotated here by 3D RoPE at (the frame's
// order in the ring, h, w); queries at (their own frame's order, h, w) --
// KV-cache relative RoPE, "NVlabs LongLive" (refft.com), Core Analysis block
// "How do KV-cache relative RoPE and TriAttention work together".  The cached
// K/V are NVFP4 ("NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long
// video generation", section "NVFP4, sequence parallel and the async decode
// path": FP4 KV dequantization and fused RoPE).
//
// Structure.  A cluster of two CTAs (one per SM) owns a pair of 128-row query
// tiles of one (b, h) at a time; key tiles are 128 keys.  Every MMA is a
// pair MMA (tcgen05 cta_group::2, M = 256) issued by the even CTA: each SM
// computes its own 128 rows and holds half of each B operand, so each SM
// dequantizes only half of every key tile:
//   K: keys [64r, 64r+64) of the tile (all 128 channels),
//   V: channels [64r, 64r+64) of all 128 keys   (r = CTA rank in the pair).
// Per CTA, 16 warps:
//   warps 0-3    softmax: thread r owns query row r = TMEM lane r.  Per tile
//                one pass over the 128 logits in TMEM in chunks of 32 (the
//                chunk's max, then its exponentials), P (f16) written back
//                over S; online softmax with lazy rescale of O (when the row
//                max grows by more than 2^8).
//   warps 4-7    K converters (two threads per key) and, per work segment,
//                the RoPE-rotated Q tile into TMEM.
//   warps 8-11   V converters (one thread per key).
//   warp 12      producer: bulk async copies (TMA engine) of the packed code
//                and scale rows into a 4-stage staging ring (NVFP4 only).
//   warp 13      TMEM allocation (both CTAs) and, in the even CTA, the MMA
//                issuer: S = Q K^T into one of two S buffers while the softmax
//                reads the other, then O += P V.  In the odd CTA its lane 0
//                relays the P and O-free events to the even CTA.
//   warps 14-15  odd CTA only: lane 0 relays the Q/K and the V events.
// TMEM per CTA: Q (64 cols, f16 pairs) | S0 (128) | S1 (128) | O (128).
// Dequantized values are exact in f16 (E2M1 code x E4M3 scale); the global
// scales fold into the softmax scale (K) and the epilogue (V).
//
// Scheduling: the grid is persistent (one CTA pair per slot).  The (b, h,
// pair) work items are laid end to end in tiles and cut into equal
// contiguous ranges, one per slot; an item cut by a range boundary is
// finished by several slots, which leave partial (O, max, sum) records in the
// workspace and the last one to finish merges them.
// Every mbarrier wait is bounded; on expiry the pair records NVKV_ERR_TIMEOUT
// in the status word, unwinds, waits for its own MMAs and frees TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nvkv_internal.h"
#include "ptx.cuh"

namespace nvkv {
namespace {

constexpr int BM = 128;                // query rows per CTA (the pair covers 256)
constexpr int BN = 128;                // keys per tile
constexpr int NTHREADS = 512;
constexpr int NSTAGE = 4;              // staging ring depth
constexpr int MAX_SEG = 96;            // work segments per slot
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait
constexpr int PAIRS_F = 22, PAIRS_H = 21, PAIRS_W = 21;   // 44 / 42 / 42 channels

constexpr uint32_t K_TILE = 16384;      // 64 keys x 128 ch f16, K-major, 128-B swizzle
constexpr uint32_t K_HALF = 8192;       // one 64-channel half of it
constexpr uint32_t V_TILE = 16384;      // 128 keys x 64 ch f16, MN-major, 128-B swizzle
constexpr uint32_t OFF_K = 0;                         // two buffers
constexpr uint32_t OFF_V = OFF_K + 2 * K_TILE;        // two buffers
constexpr uint32_t OFF_STG = OFF_V + 2 * V_TILE;      // staging ring
constexpr uint32_t STG_KC = 0, STG_KS = 4096, STG_VC = 4608, STG_VS = 12800;
constexpr uint32_t STG_BYTES = 13824;
constexpr uint32_t OFF_TAB = OFF_STG + NSTAGE * STG_BYTES;   // RoPE tables

// TMEM columns
constexpr uint32_t TM_Q = 0;      // f16 pairs of the 128 channels
constexpr uint32_t TM_S = 64;     // S buffers at 64 and 192 (f32); P over S
constexpr uint32_t TM_O = 320;    // f32

constexpr int PART_FLOATS = 130;  // O (128) + max + sum per row of a partial record

enum Bar {
    B_QREADY = 0,                         // [even CTA] both Q tiles in TMEM (256)
    B_KFULL = 1,                          // [even] + buffer: K halves (256)
    B_VFULL = 3,                          // [even] + buffer: V halves (256)
    B_P = 5,                              // [even] + buffer: P of both tiles (256)
    B_OFREE = 7,                          // [even] epilogues read O (256)
    B_S = 8,                              // + buffer: S written (commit)
    B_KFREE = 10,                         // + buffer (commit)
    B_VFREE = 12,                         // + buffer (commit)
    B_QFREE = 14,                         // segment's last S done (commit)
    B_ODONE = 15,                         // segment's last PV done (commit)
    B_MMADONE = 16,                       // everything issued is done (commit)
    B_STG_FULL = 17,                      // + stage (producer, 1 + bytes)
    B_STG_EMPTY = B_STG_FULL + NSTAGE,    // + stage (K and V converters, 256)
    N_BARS = B_STG_EMPTY + NSTAGE
};

struct Segment {
    int b, h, p;        // work item: batch, head, query tile pair
    int t0, t1;         // key tiles [t0, t1) of the item
    int n_chunks;       // slots sharing the item (1: this segment finishes it)
    int part;           // partial record index of this segment
    int first_slot;     // slot holding the item's first chunk (counter index)
    int item_start;     // flattened tile index of the item's tile 0
};

struct SharedCtl {
    uint64_t bar[N_BARS];
    int abort;
    uint32_t tmem_base;
    int n_seg;
    int merge_flag;
    float qinv[BM];     // per query row of the segment: 2^-e of its Q range scaling
    Segment seg[MAX_SEG];
};

// byte offset of 16-byte chunk c (0..15) of key row r (0..63) in a K tile
__device__ __forceinline__ uint32_t swz_k(int r, int c)
{
    return (uint32_t)((c >> 3) * K_HALF + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// byte offset of 16-byte chunk c (0..7, channels 8c..8c+7) of key k in a V tile
__device__ __forceinline__ uint32_t swz_v(int k, int c)
{
    return (uint32_t)(k * 128 + ((c ^ (k & 7)) << 4));
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint4 ldg16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void sts16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                      uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint4 lds16(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr));
    return r;
}

__device__ __forceinline__ uint2 lds8(uint32_t addr)
{
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t lds4(uint32_t addr)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    return r;
}

// four E2M1 pairs (one 32-bit word of codes) -> four f16x2 (low nibble low)
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t *h)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

// one E4M3 byte -> (v, v) as f16x2 (exact)
__device__ __forceinline__ __half2 e4m3_to_h2(uint32_t byte)
{
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)(byte | (byte << 8))));
    return *reinterpret_cast<__half2 *>(&r);
}

__device__ __forceinline__ __half2 as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }
__device__ __forceinline__ uint32_t as_u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// Both caches feed the tensor cores f16 operands (kind::f16, f32 accumulate).
// NVFP4: code * s_b is exact in f16.  bf16 twin: cached values convert to f16
// exactly inside f16's normal range (|x| in [2^-14, 65504]); rotated keys,
// queries and probabilities keep 3 more mantissa bits than bf16 would.
constexpr uint32_t kOperandF16 = 0;

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi)
{
    return as_u(__floats2half2_rn(lo, hi));
}

// x / d for 0 <= x < 2^24 by a float reciprocal with a one-step fix-up
__device__ __forceinline__ int div_fast(int x, int d, float inv)
{
    int q = __float2int_rz((float)x * inv);
    if (q * d > x) --q;
    else if ((q + 1) * d <= x) ++q;
    return q;
}

struct Ctx {
    const AttnLaunch *a;
    uint8_t *smem;
    SharedCtl *ctl;
    uint32_t sbase;                 // shared-space address of smem
    uint32_t tab_f, tab_h, tab_w;   // byte offsets of the three RoPE tables
    uint32_t rank;                  // CTA rank in the pair
    uint32_t lead_bar;              // shared::cluster address of the even CTA's bar[0]
    uint32_t peer_abort;            // shared::cluster address of the other CTA's abort flag
    int slot;
};

__device__ __forceinline__ uint32_t lead(const Ctx &c, int bar) { return c.lead_bar + bar * 8; }

__device__ __forceinline__ void set_abort(Ctx &c)
{
    if (atomicExch(&c.ctl->abort, 1) == 0) {
        atomicCAS(c.a->status, 0, (int)NVKV_ERR_TIMEOUT);
        ptx::st_cluster_u32(c.peer_abort, 1u);
    }
}

__device__ __forceinline__ bool wait(Ctx &c, int bar, uint32_t parity)
{
    if (ptx::mbar_wait(&c.ctl->bar[bar], parity, &c.ctl->abort, WAIT_LIMIT_NS)) return true;
    set_abort(c);
    return false;
}

// Cross-CTA events (Q ready, K/V halves converted, P written, O read) are
// counted on the even CTA's barrier.  Every thread arrives on its own CTA's
// copy; in the odd CTA one relay thread per event stream waits for the local
// phase and forwards it with a single remote arrive.  All arrives release and
// all waits acquire at CTA scope: what an event publishes is in the
// publishing CTA's own shared memory (made visible to the tensor core by
// fence.proxy.async) or TMEM (ordered by the tcgen05 thread-sync fences), and
// the peer reads it only through the pair MMA issued after the wait.  A
// cluster-scope release or acquire costs hundreds of cycles per event here
// and lengthens the P -> PV -> S -> softmax loop by as much.
__device__ __forceinline__ void arrive_x(Ctx &c, int bar) { ptx::mbar_arrive(&c.ctl->bar[bar]); }

// wait by every lane of a warp, outcome made warp-uniform (the tcgen05 loads
// and stores that follow are warp-collective)
__device__ __forceinline__ bool wait_warp(Ctx &c, int bar, uint32_t parity)
{
    const bool ok = wait(c, bar, parity);
    return __all_sync(0xFFFFFFFFu, ok);
}

// ------------------------------------------------------------ schedule

__device__ __forceinline__ int key_tiles(const AttnLaunch &a, int b)
{
    return (a.n_vis[b] * a.Tr + BN - 1) / BN;
}

__device__ __forceinline__ long long total_tiles(const AttnLaunch &a)
{
    long long total = 0;
    for (int b = 0; b < a.B; ++b) total += (long long)a.H * a.n_pairs * key_tiles(a, b);
    return total;
}

// The persistent schedule.  Work items are (b, h, p) in that order, item i
// of batch b taking key_tiles(b) tiles.  When every item has the same number
// of tiles, the first `rounds` * n_slots items go round-robin: slot s takes
// items s, s + n_slots, s + 2 n_slots, ...  All slots start a round together
// on neighbouring items, i.e. on the query-tile pairs of the same few heads,
// which then read each K/V tile at about the same time, so that it crosses
// HBM about once.  The remaining tiles (all of them when the items differ in
// length, as in a batch of multi-shot streams) are laid end to end and cut
// into n_slots equal ranges (stream-K); only those ranges can split an item,
// whose chunks then merge through partial records.  `rounds` stops one short
// of items / n_slots; a tail of fewer than n_slots items would be split into
// many chunks each, whose merges at the very end cost more than the rounds
// save (7 % on the 1.3B-like step).
struct TailPlan {
    int rounds;           // whole items per slot, round-robin
    long long start;      // first tile of the end-to-end part (all items laid end to end)
    long long total;      // tiles of the end-to-end part
    long long target;     // tiles per slot in it
};

__device__ __forceinline__ TailPlan tail_plan(const AttnLaunch &a)
{
    const int nkt0 = key_tiles(a, 0);
    bool uniform = true;
    for (int b = 1; b < a.B; ++b) uniform = uniform && key_tiles(a, b) == nkt0;
    const long long items = (long long)a.B * a.H * a.n_pairs;
    TailPlan t;
    // one round fewer than fit: the end-to-end part then holds at least
    // n_slots items, so that it splits each item among about two slots (as
    // many as it would hold alone, with fewer partial records to merge at
    // the end)
    t.rounds = uniform ? max(0, (int)(items / a.n_slots) - 1) : 0;
    t.start = (long long)t.rounds * a.n_slots * nkt0;
    t.total = total_tiles(a) - t.start;
    t.target = (t.total + a.n_slots - 1) / a.n_slots;
    return t;
}

__device__ void build_schedule(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const TailPlan tp = tail_plan(a);
    const int per_b = a.H * a.n_pairs;
    int n = 0;
    for (int r = 0; r < tp.rounds && n < MAX_SEG; ++r) {
        const int item = r * a.n_slots + c.slot;
        const int b = item / per_b, hp = item - b * per_b;
        Segment &s = c.ctl->seg[n++];
        s.b = b;
        s.h = hp / a.n_pairs;
        s.p = hp - s.h * a.n_pairs;
        s.t0 = 0;
        s.t1 = key_tiles(a, b);
        s.n_chunks = 1;
        s.first_slot = c.slot;
        s.item_start = 0;
        s.part = 0;
    }
    const long long beg = tp.start + (long long)c.slot * tp.target;
    const long long end = min(tp.start + tp.total, beg + tp.target);
    long long u = beg;
    long long base = 0;
    for (int b = 0; b < a.B && u < end; ++b) {
        const int nkt = key_tiles(a, b);
        const long long span = (long long)per_b * nkt;
        while (u < end && u < base + span && n < MAX_SEG) {
            const long long off = u - base;
            const int item = (int)(off / nkt);
            const int t0 = (int)(off - (long long)item * nkt);
            // the item's first tile, counted from the start of the end-to-end part
            const long long item_start = base + (long long)item * nkt - tp.start;
            const long long seg_end = min(end, tp.start + item_start + nkt);
            Segment &s = c.ctl->seg[n++];
            s.b = b;
            s.h = item / a.n_pairs;
            s.p = item - s.h * a.n_pairs;
            s.t0 = t0;
            s.t1 = t0 + (int)(seg_end - u);
            const int first = (int)(item_start / tp.target);
            const int last = (int)((item_start + nkt - 1) / tp.target);
            s.n_chunks = last - first + 1;
            s.first_slot = first;
            s.item_start = (int)item_start;
            s.part = 2 * c.slot + (u == beg ? 0 : 1);
            u = seg_end;
        }
        base += span;
    }
    c.ctl->n_seg = n;
}

// partial record index of chunk k of an item (see build_schedule)
__device__ __forceinline__ int chunk_part(const Segment &s, int k, long long target)
{
    const int slot = s.first_slot + k;
    return 2 * slot + ((k == 0 && (long long)s.item_start > (long long)slot * target) ? 1 : 0);
}

// ------------------------------------------------------------ RoPE tables

// Entry (pos, pair): NVFP4 path (c, c) and (-s, s) as f16x2; bf16 twin (c, s)
// as f32.  Angle = pos * theta[pair] with theta from the host in double.
template <bool FP4>
__device__ void build_tables(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const int nf = a.n_fpos * PAIRS_F, nh = a.grid_h * PAIRS_H, nw = a.grid_w * PAIRS_W;
    for (int i = threadIdx.x; i < nf + nh + nw; i += NTHREADS) {
        int pos, p;
        uint32_t off;
        if (i < nf) {
            pos = i / PAIRS_F; p = i % PAIRS_F; off = c.tab_f + i * 8;
        } else if (i < nf + nh) {
            const int k = i - nf;
            pos = k / PAIRS_H; p = PAIRS_F + k % PAIRS_H; off = c.tab_h + k * 8;
        } else {
            const int k = i - nf - nh;
            pos = k / PAIRS_W; p = PAIRS_F + PAIRS_H + k % PAIRS_W; off = c.tab_w + k * 8;
        }
        float sn, cs;
        sincosf((float)pos * a.theta[p], &sn, &cs);
        uint32_t *e = reinterpret_cast<uint32_t *>(c.smem + off);
        if (FP4) {
            e[0] = as_u(__floats2half2_rn(cs, cs));
            e[1] = as_u(__floats2half2_rn(-sn, sn));
        } else {
            e[0] = __float_as_uint(cs);
            e[1] = __float_as_uint(sn);
        }
    }
}

// Row bases of the three tables for a token at (frame position fpos, row hp,
// column wp), pre-offset so that the entry of channel pair p is at
// base(axis of p) + 8 p.
struct RopeRows {
    uint32_t f, h, w;
};

__device__ __forceinline__ RopeRows rope_rows(const Ctx &c, int fpos, int hp, int wp)
{
    RopeRows rr;
    rr.f = c.sbase + c.tab_f + fpos * (PAIRS_F * 8);
    rr.h = c.sbase + c.tab_h + hp * (PAIRS_H * 8) - PAIRS_F * 8;
    rr.w = c.sbase + c.tab_w + wp * (PAIRS_W * 8) - (PAIRS_F + PAIRS_H) * 8;
    return rr;
}

// shared address of pair p's entry (p is a constant after unrolling)
__device__ __forceinline__ uint32_t rope_at(const RopeRows &rr, int p)
{
    return (p < PAIRS_F ? rr.f : p < PAIRS_F + PAIRS_H ? rr.h : rr.w) + p * 8;
}

struct KeyPos {
    bool valid;
    RopeRows rr;
    size_t grow;   // global row index into the [B][H][R] planes
};

// Keys are numbered Tr per visible frame: key f Tr + i is row i of frame f's
// slot, a token for i < Tk and the padding row (invalid) for i = Tk.
// tok_off: index within the frame of the cache's first token (a shard of a
// sequence-parallel KV split), a constant 0 for a whole cache.
__device__ __forceinline__ KeyPos key_pos(const Ctx &c, int b, int h, int n_keys, int key,
                                          int tok_off)
{
    const AttnLaunch &a = *c.a;
    KeyPos k;
    const int kk = key < n_keys ? key : 0;
    const int f = div_fast(kk, a.Tr, a.inv_Tr);
    const int tok = kk - f * a.Tr;
    k.valid = key < n_keys && tok < a.Tk;
    const VisFrame vf = a.vis[b][f];
    const int ft = tok_off + min(tok, a.Tk - 1);   // the token's index in its frame
    const int hp = div_fast(ft, a.grid_w, a.inv_grid_w);
    k.rr = rope_rows(c, vf.rope_pos, hp, ft - hp * a.grid_w);
    k.grow = (size_t)(b * a.H + h) * a.R + (size_t)vf.slot * a.Tr + tok;
    return k;
}

// 0 for the padding key of an odd shard (key mod Tr == Tk), else 1
__device__ __forceinline__ bool not_pad(const AttnLaunch &a, int key)
{
    const int f = div_fast(key, a.Tr, a.inv_Tr);
    return key - f * a.Tr < a.Tk;
}

// ------------------------------------------------------------ Q prologue

// Q row `row` of the chunk -> times 2^e -> RoPE in f32 -> f16 pairs in TMEM
// columns [tcol, tcol + 64) of this thread's lane; 2^-e is returned in
// qinv_out.  e puts the row's largest |q| in [2^13, 2^14), so that the
// rotated row (|rot| <= sqrt(2) max |q|) lies inside f16's normal range for
// any finite bf16 input; the softmax multiplies its logit scale by 2^-e.  A
// power of two commutes exactly with the f16 rounding (normal range), the
// products and the f32 sums of S = Q K^T, so for rows already inside the
// range the logits are unchanged bit for bit.  The row is read twice (its
// max, then the values), the second time from L1.
template <bool FP4>
__device__ void load_q_tmem(const Ctx &c, int b, int h, int row, uint32_t tcol, float &qinv_out)
{
    const AttnLaunch &a = *c.a;
    const bool valid = row < a.Lq;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.q) +
                       (((size_t)b * a.Lq + (valid ? row : 0)) * a.H + h) * 16;
    const int frame = valid ? div_fast(row, a.T, a.inv_T) : 0;
    const int tok = valid ? row - frame * a.T : 0;
    const int hp = div_fast(tok, a.grid_w, a.inv_grid_w);
    const RopeRows rr = rope_rows(c, a.q_pos0[b] + frame, hp, tok - hp * a.grid_w);
    uint32_t mx = 0;                           // max |bf16| bits, both halves
    if (valid) {
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
            const uint4 w = ldg16(src + ch);
            mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu),
                                       __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
        }
    }
    mx = max(mx >> 16, mx & 0xFFFFu);          // bf16 bits of max |q|
    // e = 13 - floor(log2 max |q|), from the biased exponent; 0 for a zero row
    // (or one holding infinities or NaN); kept inside [-126, 126]
    const int ebits = (int)((mx >> 7) & 0xFFu);
    int e = (mx == 0 || ebits == 0xFF) ? 0 : 140 - ebits;
    e = max(-126, min(126, e));
    const float up = __uint_as_float((uint32_t)(127 + e) << 23);
    qinv_out = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 wv = valid ? ldg16(src + hh * 8 + ch) : make_uint4(0, 0, 0, 0);
            const uint32_t u[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int p = hh * 32 + ch * 4 + k;
                const float x = __uint_as_float(u[k] << 16) * up;
                const float y = __uint_as_float(u[k] & 0xFFFF0000u) * up;
                const uint2 e2 = lds8(rope_at(rr, p));
                float cs, sn;
                if (FP4) {
                    cs = __low2float(as_h2(e2.x));
                    sn = __high2float(as_h2(e2.y));
                } else {
                    cs = __uint_as_float(e2.x);
                    sn = __uint_as_float(e2.y);
                }
                o[ch * 4 + k] = pack_f16(x * cs - y * sn, x * sn + y * cs);
            }
        }
        ptx::tmem_st32(tcol + hh * 32, o);
    }
}

// ------------------------------------------------------------ converters

// K, NVFP4: staging key row sr (0..63), channel half HH (pairs 32HH ..
// 32HH+31) into row sr of the K tile: decode, scale (exact), rotate.  An
// invalid key reads zero codes and writes zeros.
template <int HH>
__device__ __forceinline__ void conv_k_fp4(uint32_t stg, int sr, const KeyPos &k, uint32_t kdst)
{
    uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
    uint32_t sc = 0;
    if (k.valid) {
        w0 = lds16(stg + STG_KC + sr * 64 + HH * 32);
        w1 = lds16(stg + STG_KC + sr * 64 + HH * 32 + 16);
        sc = lds4(stg + STG_KS + sr * 8 + HH * 4);
    }
    const uint32_t code[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {          // output chunk 8HH + cc
        const __half2 sb = e4m3_to_h2((sc >> (8 * (cc >> 1))) & 0xFFu);
        uint32_t hq[4], o[4];
        e2m1x8_to_f16(code[cc], hq);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = (HH * 8 + cc) * 4 + q;
            const __half2 v = __hmul2(as_h2(hq[q]), sb);          // (x, y) * s_b, exact
            const uint2 e = lds8(rope_at(k.rr, p));
            // (x c - y s, y c + x s)
            o[q] = as_u(__hfma2(__lowhigh2highlow(v), as_h2(e.y), __hmul2(v, as_h2(e.x))));
        }
        sts16(kdst + swz_k(sr, HH * 8 + cc), o[0], o[1], o[2], o[3]);
    }
}

// V, NVFP4: staging key row k (0..127), this CTA's channel half (bytes
// [32 half, 32 half + 32) of the packed row, scale blocks 4 half .. +3).
__device__ __forceinline__ void conv_v_fp4(uint32_t stg, int k, int half, bool valid,
                                           uint32_t vdst)
{
    uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
    uint32_t sc = 0;
    if (valid) {
        w0 = lds16(stg + STG_VC + k * 64 + half * 32);
        w1 = lds16(stg + STG_VC + k * 64 + half * 32 + 16);
        sc = lds4(stg + STG_VS + k * 8 + half * 4);
    }
    const uint32_t code[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {          // channels 8cc .. 8cc+7 of the half
        const __half2 sb = e4m3_to_h2((sc >> (8 * (cc >> 1))) & 0xFFu);
        uint32_t hq[4];
        e2m1x8_to_f16(code[cc], hq);
        sts16(vdst + swz_v(k, cc), as_u(__hmul2(as_h2(hq[0]), sb)),
              as_u(__hmul2(as_h2(hq[1]), sb)), as_u(__hmul2(as_h2(hq[2]), sb)),
              as_u(__hmul2(as_h2(hq[3]), sb)));
    }
}

// K, bf16 twin: channel half HH of key k from global memory, RoPE in f32.
template <int HH>
__device__ __forceinline__ void conv_k_bf16(const Ctx &c, int sr, const KeyPos &k, uint32_t kdst)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(c.a->k_data) + k.grow * 16 + HH * 8;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const uint4 w = k.valid ? ldg16(src + cc) : make_uint4(0, 0, 0, 0);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = (HH * 8 + cc) * 4 + q;
            const float x = __uint_as_float(u[q] << 16), y = __uint_as_float(u[q] & 0xFFFF0000u);
            const uint2 e = lds8(rope_at(k.rr, p));
            const float cs = __uint_as_float(e.x), sn = __uint_as_float(e.y);
            o[q] = pack_f16(x * cs - y * sn, x * sn + y * cs);
        }
        sts16(kdst + swz_k(sr, HH * 8 + cc), o[0], o[1], o[2], o[3]);
    }
}

// V, bf16 twin: this CTA's channel half of key k from global memory.
__device__ __forceinline__ void conv_v_bf16(const Ctx &c, int kk, int half, const KeyPos &k,
                                            uint32_t vdst)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(c.a->v_data) + k.grow * 16 + half * 8;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const uint4 w = k.valid ? ldg16(src + cc) : make_uint4(0, 0, 0, 0);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = pack_f16(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xFFFF0000u));
        sts16(vdst + swz_v(kk, cc), o[0], o[1], o[2], o[3]);
    }
}

// warps 4-7: per segment the Q tile into TMEM, then K halves of the tiles
template <bool FP4, bool SHARD>
__device__ void k_converter_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const int t = threadIdx.x - 128;          // 0..127, TMEM lane t
    const uint32_t lane_off = (uint32_t)(t & ~31) << 16;
    const uint32_t tmem = c.ctl->tmem_base;
    const int sr = t & 63, hh = t >> 6;       // staging key row, channel half (warp-uniform)
    int g = 0;                                 // tiles processed by this CTA
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        const int n_keys = a.n_vis[sg.b] * a.Tr;
        if (si > 0 && !wait_warp(c, B_QFREE, (si - 1) & 1)) return;
        ptx::tc_fence_after();
        float qi;
        load_q_tmem<FP4>(c, sg.b, sg.h, (2 * sg.p + (int)c.rank) * BM + t,
                         tmem + lane_off + TM_Q, qi);
        c.ctl->qinv[t] = qi;                  // published by the QREADY arrive
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        arrive_x(c, B_QREADY);
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g) {
            const int s = g % NSTAGE, kb = g & 1;
            const uint32_t stg = c.sbase + OFF_STG + s * STG_BYTES;
            const uint32_t kdst = c.sbase + OFF_K + kb * K_TILE;
            const KeyPos k = key_pos(c, sg.b, sg.h, n_keys, tile * BN + 64 * (int)c.rank + sr,
                                     SHARD ? a.tok_off : 0);
            if (FP4 && !wait(c, B_STG_FULL + s, (g / NSTAGE) & 1)) return;
            if (g >= 2 && !wait(c, B_KFREE + kb, ((g - 2) >> 1) & 1)) return;
            if (FP4) {
                if (hh == 0) conv_k_fp4<0>(stg, sr, k, kdst);
                else conv_k_fp4<1>(stg, sr, k, kdst);
            } else {
                if (hh == 0) conv_k_bf16<0>(c, sr, k, kdst);
                else conv_k_bf16<1>(c, sr, k, kdst);
            }
            ptx::fence_proxy_async_smem();
            arrive_x(c, B_KFULL + kb);
            if (FP4) ptx::mbar_arrive(&c.ctl->bar[B_STG_EMPTY + s]);
        }
    }
}

// warps 8-11: this CTA's channel half of V for all 128 keys of each tile
template <bool FP4, bool SHARD, bool PAD>
__device__ void v_converter_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const int k = threadIdx.x - 256;          // key of the tile, 0..127
    int g = 0;
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        const int n_keys = a.n_vis[sg.b] * a.Tr;
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g) {
            const int s = g % NSTAGE, vb = g & 1;
            const uint32_t stg = c.sbase + OFF_STG + s * STG_BYTES;
            const uint32_t vdst = c.sbase + OFF_V + vb * V_TILE;
            if (FP4 && !wait(c, B_STG_FULL + s, (g / NSTAGE) & 1)) return;
            if (g >= 2 && !wait(c, B_VFREE + vb, ((g - 2) >> 1) & 1)) return;
            if (FP4) {
                conv_v_fp4(stg, k, (int)c.rank,
                           tile * BN + k < n_keys && (!PAD || not_pad(a, tile * BN + k)), vdst);
            } else {
                const KeyPos kp = key_pos(c, sg.b, sg.h, n_keys, tile * BN + k, SHARD ? a.tok_off : 0);
                conv_v_bf16(c, k, (int)c.rank, kp, vdst);
            }
            ptx::fence_proxy_async_smem();
            arrive_x(c, B_VFULL + vb);
            if (FP4) ptx::mbar_arrive(&c.ctl->bar[B_STG_EMPTY + s]);
        }
    }
}

// ------------------------------------------------------------ relays (odd CTA)

__device__ __forceinline__ bool relay(Ctx &c, int bar, uint32_t parity)
{
    if (!wait(c, bar, parity)) return false;
    ptx::mbar_arrive_remote(lead(c, bar));
    return true;
}

// Q and K halves, in the order the K converters produce them
__device__ void relay_qk_role(Ctx &c)
{
    int g = 0;
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        if (!relay(c, B_QREADY, si & 1)) return;
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g)
            if (!relay(c, B_KFULL + (g & 1), (g >> 1) & 1)) return;
    }
}

__device__ void relay_v_role(Ctx &c)
{
    int g = 0;
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g)
            if (!relay(c, B_VFULL + (g & 1), (g >> 1) & 1)) return;
    }
}

// P of every tile, then O released at the end of each segment
__device__ void relay_p_role(Ctx &c)
{
    int g = 0;
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g)
            if (!relay(c, B_P + (g & 1), (g >> 1) & 1)) return;
        if (!relay(c, B_OFREE, si & 1)) return;
    }
}

// ------------------------------------------------------------ producer

// Bulk copies of one tile's packed rows: this CTA's 64 K rows and all 128 V
// rows.  Every run of consecutive keys inside one frame is contiguous in the
// planes; run starts and lengths are even (Tr even, tiles of 64 keys), so every copy is 16-byte
// aligned and sized.
__device__ __forceinline__ void copy_runs(const AttnLaunch &a, int b, size_t head_row0, int k0,
                                          int k1, uint8_t *dst_c, uint8_t *dst_s,
                                          const uint8_t *codes, const uint8_t *scales,
                                          uint64_t *full)
{
    for (int k = k0; k < k1;) {
        const int f = div_fast(k, a.Tr, a.inv_Tr), tok = k - f * a.Tr;
        const int n = min(a.Tr - tok, k1 - k);
        const size_t g = head_row0 + (size_t)a.vis[b][f].slot * a.Tr + tok;
        const int t0 = k - k0;
        ptx::bulk_g2s(dst_c + t0 * 64, codes + g * 64, (uint32_t)n * 64, full);
        ptx::bulk_g2s(dst_s + t0 * 8, scales + g * 8, (uint32_t)n * 8, full);
        k += n;
    }
}

// FAULT: the failure-path test variant (nvkv_debug_inject_fault): the first
// stage is never filled, so the waits on it run out
template <bool FAULT>
__device__ void producer_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    int g = 0;
    bool ok = true;
    for (int si = 0; ok && si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        const int n_keys = a.n_vis[sg.b] * a.Tr;
        const size_t head_row0 = (size_t)(sg.b * a.H + sg.h) * a.R;
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g) {
            const int s = g % NSTAGE;
            if (g >= NSTAGE && !(ok = wait(c, B_STG_EMPTY + s, ((g - NSTAGE) / NSTAGE) & 1)))
                break;
            if (FAULT && g == 0) continue;
            uint8_t *stg = c.smem + OFF_STG + s * STG_BYTES;
            uint64_t *full = &c.ctl->bar[B_STG_FULL + s];
            const int kk0 = min(n_keys, tile * BN + 64 * (int)c.rank);
            const int kk1 = min(n_keys, tile * BN + 64 * (int)c.rank + 64);
            const int vk0 = tile * BN;
            const int vk1 = min(n_keys, vk0 + BN);
            ptx::mbar_arrive_expect_tx(full, (uint32_t)((kk1 - kk0) + (vk1 - vk0)) * 72u);
            copy_runs(a, sg.b, head_row0, kk0, kk1, stg + STG_KC, stg + STG_KS,
                      static_cast<const uint8_t *>(a.k_data),
                      static_cast<const uint8_t *>(a.k_scales), full);
            copy_runs(a, sg.b, head_row0, vk0, vk1, stg + STG_VC, stg + STG_VS,
                      static_cast<const uint8_t *>(a.v_data),
                      static_cast<const uint8_t *>(a.v_scales), full);
        }
    }
    // no CTA leaves with copies into its shared memory in flight (after an
    // abort, stages nobody consumed may still be landing)
    const int never = 0;
    for (int i = g - 1; i >= 0 && i >= g - NSTAGE; --i) {
        if (FAULT && i == 0) continue;
        ptx::mbar_wait(&c.ctl->bar[B_STG_FULL + i % NSTAGE], (i / NSTAGE) & 1, &never,
                       WAIT_LIMIT_NS);
    }
}

// ------------------------------------------------------------ MMA issuer

__device__ void mma_role(Ctx &c)
{
    const uint32_t tmem = c.ctl->tmem_base;
    constexpr uint32_t idS = ptx::idesc_f16(kOperandF16, 2 * BM, BN, 0);
    constexpr uint32_t idO = ptx::idesc_f16(kOperandF16, 2 * BM, 128, 1);
    const uint32_t ks = c.sbase + OFF_K;
    const uint32_t vs = c.sbase + OFF_V;
    const uint16_t both = 0x3;

    // Shared-memory descriptors: the start address (>> 4) is the low field,
    // so the descriptor of base + off is desc(base) + off / 16 (all of shared
    // memory lies below 2^18 bytes, so the field cannot carry).  Built once,
    // they leave the issuing thread two adds per MMA.
    const uint64_t dk0 = ptx::smem_desc_sw128(ks, 16, 1024);
    const uint64_t dv0 = ptx::smem_desc_sw128(vs, V_TILE, 1024);
    // S_buf = Q K^T: A = Q (TMEM, 8 x 16 channels), B = the K halves, K-major
    auto issue_s = [&](int buf, int kb) {
        const uint64_t dk = dk0 + (uint64_t)(kb * (K_TILE >> 4));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            ptx::mma2_f16_ts(tmem + TM_S + buf * 128, tmem + TM_Q + kk * 8,
                             dk + (uint64_t)(((kk >> 2) * K_HALF + (kk & 3) * 32) >> 4), idS,
                             kk > 0);
        ptx::mma2_commit_mc(&c.ctl->bar[B_S + buf], both);
        ptx::mma2_commit_mc(&c.ctl->bar[B_KFREE + kb], both);
    };
    // O += P V: A = P (TMEM over S_buf, 8 x 16 keys), B = the V halves, MN-major
    auto issue_pv = [&](int buf, int vb, bool first) {
        const uint64_t dv = dv0 + (uint64_t)(vb * (V_TILE >> 4));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            ptx::mma2_f16_ts(tmem + TM_O, tmem + TM_S + buf * 128 + kk * 8,
                             dv + (uint64_t)(kk * (2048 >> 4)), idO, (!first || kk > 0) ? 1u : 0u);
        ptx::mma2_commit_mc(&c.ctl->bar[B_VFREE + vb], both);
    };

    int g = 0;
    bool ok = true;
    for (int si = 0; ok && si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        const int n = sg.t1 - sg.t0, g0 = g;
        if (!(ok = wait(c, B_QREADY, si & 1) && wait(c, B_KFULL + (g0 & 1), (g0 >> 1) & 1)))
            break;
        ptx::tc_fence_after();
        issue_s(g0 & 1, g0 & 1);
        for (int i = 0; i < n; ++i, ++g) {
            if (i + 1 < n) {
                if (!(ok = wait(c, B_KFULL + ((g + 1) & 1), ((g + 1) >> 1) & 1))) break;
                ptx::tc_fence_after();
                issue_s((g + 1) & 1, (g + 1) & 1);
            }
            if (!(ok = wait(c, B_VFULL + (g & 1), (g >> 1) & 1) &&
                       wait(c, B_P + (g & 1), (g >> 1) & 1) &&
                       (i > 0 || si == 0 || wait(c, B_OFREE, (si - 1) & 1))))
                break;
            ptx::tc_fence_after();
            issue_pv(g & 1, g & 1, i == 0);
        }
        if (!ok) break;
        ptx::mma2_commit_mc(&c.ctl->bar[B_QFREE], both);
        ptx::mma2_commit_mc(&c.ctl->bar[B_ODONE], both);
    }
    // every MMA issued has finished (in both CTAs) before TMEM is released
    ptx::mma2_commit_mc(&c.ctl->bar[B_MMADONE], both);
}

// ------------------------------------------------------------ softmax

__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha)
{
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        ptx::tmem_ld32(tO + q * 32, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])),
                                        make_float2(alpha, alpha));
            o[i] = __float_as_uint(v.x);
            o[i + 1] = __float_as_uint(v.y);
        }
        ptx::tmem_st32(tO + q * 32, o);
    }
}

__device__ __forceinline__ void store_row_bf16(uint4 *dst, const float *acc, float fin)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 bb = __floats2bfloat162_rn(acc[8 * i + 2 * k] * fin,
                                                      acc[8 * i + 2 * k + 1] * fin);
            w[k] = *reinterpret_cast<uint32_t *>(&bb);
        }
        dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <bool FP4, bool PAD>
__device__ void softmax_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const int r = threadIdx.x;                      // 0..127 = TMEM lane
    const uint32_t lane_off = (uint32_t)(r & ~31) << 16;
    const uint32_t tmem = c.ctl->tmem_base + lane_off;
    const uint32_t tO = tmem + TM_O;
    float *ws = static_cast<float *>(a.workspace);
    int *counters = reinterpret_cast<int *>(ws + (size_t)a.n_slots * 2 * 2 * BM * PART_FLOATS);
    const long long target = tail_plan(a).target;
    int g = 0;
    for (int si = 0; si < c.ctl->n_seg; ++si) {
        const Segment sg = c.ctl->seg[si];
        const int n_keys = a.n_vis[sg.b] * a.Tr;
        const int gi = sg.b * a.H + sg.h;
        const float sgk = FP4 ? a.s_g[gi] : 1.0f;
        const float sgv = FP4 ? a.s_g[a.B * a.H + gi] : 1.0f;
        // this row's Q range scaling, written with the segment's Q tile:
        // wait for that tile (its phase cannot run ahead: the next segment's
        // Q waits for this segment's last PV, which needs this thread's P)
        if (!wait_warp(c, B_QREADY, si & 1)) return;
        ptx::tc_fence_after();
        const float qinv = c.ctl->qinv[r];
        // log2(e)/sqrt(128) times s_g(K) times the row's 2^-e (all exact
        // powers of two but the first)
        const float scale = sgk * 1.4426950408889634f * 0.08838834764831845f * qinv;
        float m = -INFINITY, l = 0.0f;
        for (int tile = sg.t0; tile < sg.t1; ++tile, ++g) {
            const int buf = g & 1;
            if (!wait_warp(c, B_S + buf, (g >> 1) & 1)) return;
            ptx::tc_fence_after();
            const uint32_t tS = tmem + TM_S + buf * 128;
            const int nv = n_keys - tile * BN;   // valid keys of this tile (may exceed 128)
            // one pass: per chunk of 32 logits, its max first; a chunk whose
            // max exceeds the running max m by more than 2^8 raises m (on a
            // segment's first chunk always, rarely after), rescaling the P
            // already written in this tile, the partial sums and O
            float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            float alpha_o = 1.0f;
            bool grew = false;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                float s[32];
                ptx::tmem_ld32(tS + q * 32, reinterpret_cast<uint32_t *>(s));
                ptx::tmem_wait_ld();
                if (nv < BN) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (q * 32 + i >= nv) s[i] = -INFINITY;
                }
                if (PAD) {
                    // padding keys (one per frame, key mod Tr == Tk) of this chunk
                    const int k0 = tile * BN + q * 32;
                    uint32_t pad = 0;
                    for (int i = a.Tk - (k0 - div_fast(k0, a.Tr, a.inv_Tr) * a.Tr); i < 32;
                         i += a.Tr)
                        if (i >= 0) pad |= 1u << i;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if ((pad >> i) & 1u) s[i] = -INFINITY;
                }
                float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int i = 4; i < 32; ++i) mx4[i & 3] = fmaxf(mx4[i & 3], s[i]);
                const float cm = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale;
                if (__any_sync(0xFFFFFFFFu, cm > m + 8.0f)) {
                    const float mn = fmaxf(m, cm);
                    const float al = ex2(m - mn);          // 0 while m is -inf
                    m = mn;
                    l *= al;
                    alpha_o *= al;
                    grew = true;
                    acc[0] = __fmul2_rn(acc[0], make_float2(al, al));
                    acc[1] = __fmul2_rn(acc[1], make_float2(al, al));
                    if (q > 0) {
                        ptx::tmem_wait_st();
                        for (int k = 0; k < q; ++k) {
                            uint32_t v[16];
                            ptx::tmem_ld16(tS + k * 16, v);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float2 f = __half22float2(as_h2(v[i]));
                                v[i] = pack_f16(f.x * al, f.y * al);
                            }
                            ptx::tmem_st16(tS + k * 16, v);
                            ptx::tmem_wait_st();
                        }
                    }
                }
                const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(-m, -m);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 t2 = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), sc2, nm2);
                    const float2 p = make_float2(ex2(t2.x), ex2(t2.y));
                    acc[i & 1] = __fadd2_rn(acc[i & 1], p);
                    pk[i] = pack_f16(p.x, p.y);
                }
                ptx::tmem_st16(tS + q * 16, pk);
            }
            if (grew && tile > sg.t0) {
                // O holds the previous tile's PV once its V buffer was freed
                const int gp = g - 1;
                if (!wait_warp(c, B_VFREE + (gp & 1), (gp >> 1) & 1)) return;
                ptx::tc_fence_after();
                rescale_o(tO, alpha_o);
            }
            const float2 at = __fadd2_rn(acc[0], acc[1]);
            l += at.x + at.y;
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            arrive_x(c, B_P + buf);
        }
        // epilogue of the segment
        if (!wait_warp(c, B_ODONE, si & 1)) return;
        ptx::tc_fence_after();
        const int row = (2 * sg.p + (int)c.rank) * BM + r;
        if (sg.n_chunks == 1) {
            const float fin = sgv / l;
            uint4 *dst = reinterpret_cast<uint4 *>(a.out) +
                         (((size_t)sg.b * a.Lq + (row < a.Lq ? row : 0)) * a.H + sg.h) * 16;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                float o[32];
                ptx::tmem_ld32(tO + q * 32, reinterpret_cast<uint32_t *>(o));
                ptx::tmem_wait_ld();
                if (row < a.Lq) store_row_bf16(dst + q * 4, o, fin);
            }
            ptx::tc_fence_before();
            arrive_x(c, B_OFREE);
            if (a.lse && row < a.Lq)
                a.lse[(size_t)gi * a.Lq + row] = (m + __log2f(l)) * 0.6931471805599453f;
        } else {
            // partial record: unnormalised O, running max, sum
            float *rec = ws + (((size_t)sg.part * 2 + c.rank) * BM + r) * PART_FLOATS;
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t o[32];
                ptx::tmem_ld32(tO + q * 32, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) __stcg(rec + q * 32 + i, __uint_as_float(o[i]));
            }
            __stcg(rec + 128, m);
            __stcg(rec + 129, l);
            ptx::tc_fence_before();
            arrive_x(c, B_OFREE);
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            int *ctr = counters + 2 * sg.first_slot + c.rank;
            if (r == 0) c.ctl->merge_flag = (atomicAdd(ctr, 1) == sg.n_chunks - 1) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (c.ctl->merge_flag) {
                __threadfence();
                // merge every chunk's record for this row (this one included)
                float mm = -INFINITY;
                for (int k = 0; k < sg.n_chunks; ++k) {
                    const float *rk =
                        ws + (((size_t)chunk_part(sg, k, target) * 2 + c.rank) * BM + r) * PART_FLOATS;
                    mm = fmaxf(mm, __ldcg(rk + 128));
                }
                float wk[8];
                float lsum = 0.0f;
                const int nk = sg.n_chunks;
                for (int k = 0; k < nk && k < 8; ++k) {
                    const float *rk =
                        ws + (((size_t)chunk_part(sg, k, target) * 2 + c.rank) * BM + r) * PART_FLOATS;
                    wk[k] = ex2(__ldcg(rk + 128) - mm);
                    lsum += wk[k] * __ldcg(rk + 129);
                }
                for (int k = 8; k < nk; ++k) {
                    const float *rk =
                        ws + (((size_t)chunk_part(sg, k, target) * 2 + c.rank) * BM + r) * PART_FLOATS;
                    lsum += ex2(__ldcg(rk + 128) - mm) * __ldcg(rk + 129);
                }
                const float fin = sgv / lsum;
                uint4 *dst = reinterpret_cast<uint4 *>(a.out) +
                             (((size_t)sg.b * a.Lq + (row < a.Lq ? row : 0)) * a.H + sg.h) * 16;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    float o[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0.0f;
                    for (int k = 0; k < nk; ++k) {
                        const float *rk =
                            ws + (((size_t)chunk_part(sg, k, target) * 2 + c.rank) * BM + r) *
                                     PART_FLOATS;
                        const float w = k < 8 ? wk[k] : ex2(__ldcg(rk + 128) - mm);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = fmaf(w, __ldcg(rk + q * 32 + i), o[i]);
                    }
                    if (row < a.Lq) store_row_bf16(dst + q * 4, o, fin);
                }
                if (a.lse && row < a.Lq)
                    a.lse[(size_t)gi * a.Lq + row] = (mm + __log2f(lsum)) * 0.6931471805599453f;
                if (r == 0) *ctr = 0;      // leave the workspace zeroed
            }
        }
    }
}

// ------------------------------------------------------------ kernel

// VAR 0: a whole cache with an even number of tokens per frame; 1 (SHARD):
// a shard whose first token is not token 0 of the frame; 3: a cache whose
// slots hold a padding row (odd token count per frame), shard or not; 2: the
// failure-path test.  Separate instantiations keep the
// whole-cache kernel's code free of both.
template <bool FP4, int VAR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
    k_chunk_attn(const __grid_constant__ AttnLaunch a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctx c;
    c.a = &a;
    c.smem = smem;
    c.sbase = ptx::smem_u32(smem);
    c.rank = ptx::cluster_ctarank();
    c.slot = blockIdx.x >> 1;
    c.tab_f = OFF_TAB;
    c.tab_h = c.tab_f + a.n_fpos * PAIRS_F * 8;
    c.tab_w = c.tab_h + a.grid_h * PAIRS_H * 8;
    const uint32_t ctl_off = (c.tab_w + a.grid_w * PAIRS_W * 8 + 63) & ~63u;
    c.ctl = reinterpret_cast<SharedCtl *>(smem + ctl_off);
    c.lead_bar = ptx::mapa(ptx::smem_u32(&c.ctl->bar[0]), 0);
    c.peer_abort = ptx::mapa(ptx::smem_u32(&c.ctl->abort), c.rank ^ 1u);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        // arrival counts: a cross-CTA event takes the 128 threads of its role
        // in this CTA, plus, in the even CTA, the odd CTA's relay;
        // tcgen05.commit arrives once; staging full is the producer (1, plus
        // bytes); staging empty the K and V converters.
        for (int i = 0; i < N_BARS; ++i) {
            uint32_t n = 1;
            if (i < B_S) n = c.rank == 0 ? 129 : 128;
            if (i >= B_STG_EMPTY) n = 256;
            ptx::mbar_init(&c.ctl->bar[i], n);
        }
        c.ctl->abort = 0;
        build_schedule(c);
        ptx::fence_mbar_init();
    }
    build_tables<FP4>(c);
    if (warp == 13) {
        ptx::tmem_alloc2(&c.ctl->tmem_base, 512);
        ptx::tmem_relinquish2();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();          // peer barriers initialised before any remote arrive
    ptx::tc_fence_after();

    if (warp < 4) {
        softmax_role<FP4, VAR == 3>(c);
    } else if (warp < 8) {
        k_converter_role<FP4, VAR == 1 || VAR == 3>(c);
    } else if (warp < 12) {
        v_converter_role<FP4, VAR == 1 || VAR == 3, VAR == 3>(c);
    } else if (warp == 12) {
        if (FP4 && (threadIdx.x & 31) == 0) producer_role<VAR == 2>(c);
    } else if (warp == 13) {
        if ((threadIdx.x & 31) == 0) {
            if (c.rank == 0) mma_role(c);
            else relay_p_role(c);
        }
        __syncwarp();
        // both CTAs: every MMA touching this CTA's TMEM has completed
        const int never = 0;
        if ((threadIdx.x & 31) == 0)
            ptx::mbar_wait(&c.ctl->bar[B_MMADONE], 0, &never, WAIT_LIMIT_NS);
        __syncwarp();
    } else if (c.rank == 1 && (threadIdx.x & 31) == 0) {
        if (warp == 14) relay_qk_role(c);
        else relay_v_role(c);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();          // no CTA leaves while its peer may touch its memory
    if (warp == 13) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc2(c.ctl->tmem_base, 512);
    }
}

// dynamic shared memory of one CTA: alignment slack, operand tiles, staging,
// RoPE tables (one row per frame position, h and w), control block
uint32_t smem_bytes(const AttnLaunch &a)
{
    const uint32_t tab =
        (uint32_t)(a.n_fpos * PAIRS_F + a.grid_h * PAIRS_H + a.grid_w * PAIRS_W) * 8;
    return 1024 + OFF_TAB + ((tab + 63) & ~63u) + sizeof(SharedCtl);
}

constexpr uint32_t kMaxSmem = 232448;   // per CTA, opt-in

template <bool FP4, int VAR>
cudaError_t launch(const AttnLaunch &a, cudaStream_t s)
{
    const uint32_t bytes = smem_bytes(a);
    if (bytes > kMaxSmem) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(k_chunk_attn<FP4, VAR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid(2 * a.n_slots, 1, 1);
    k_chunk_attn<FP4, VAR><<<grid, NTHREADS, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool attention_fits(const AttnLaunch &a) { return smem_bytes(a) <= kMaxSmem; }

size_t attention_workspace_bytes(int n_slots)
{
    return (size_t)n_slots * 2 * 2 * BM * PART_FLOATS * sizeof(float) +
           (size_t)n_slots * 2 * sizeof(int);
}

int attention_slots(int device)
{
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
        return 0;
    return sms / 2;
}

cudaError_t launch_chunk_attention(const AttnLaunch &a, cudaStream_t s)
{
    const bool fp4 = a.kv_dtype == NVKV_KV_NVFP4;
    if (fp4 && a.fault == NVKV_FAULT_SKIP_FIRST_STAGE && !a.tok_off) return launch<true, 2>(a, s);
    if (a.Tr != a.Tk) return fp4 ? launch<true, 3>(a, s) : launch<false, 3>(a, s);
    if (a.tok_off) return fp4 ? launch<true, 1>(a, s) : launch<false, 1>(a, s);
    return fp4 ? launch<true, 0>(a, s) : launch<false, 0>(a, s);
}

}  // namespace nvkv
