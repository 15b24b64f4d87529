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
// Structure: one CTA per (256 query rows = Q tiles A and B, head, batch);
// key tiles of 64; 16 warps.
//   warps 0-3    softmax of Q tile A, warps 4-7 softmax of Q tile B: thread r
//                owns query row r = TMEM lane r.  Per key tile it reads its 64
//                logits once from TMEM, keeps the online softmax in registers
//                (lazy rescale of O when the row max grows by more than 2^8)
//                and writes P (f16) back into TMEM over S.
//   warps 8-11   K converters: first RoPE-rotate Q_A/Q_B into TMEM; then per
//                key tile two threads per key, each half a row: E2M1 codes ->
//                f16 by cvt, times the E4M3 block scale (exact in f16), RoPE in
//                packed f16x2 math, into a 128-byte-swizzled K-major UMMA tile.
//   warps 12-13  V converters: one thread per key: decode and scale into the
//                V tile (read by the MMA as MN-major).
//   warp 14      producer: bulk async copies (TMA engine) of each tile's packed
//                code and scale rows, run by run, into a 4-stage staging ring.
//   warp 15      TMEM allocation and the MMA issuer (one thread):
//                S = Q K^T (Q from TMEM, K from shared memory) and O += P V
//                (P from TMEM, V from shared memory), kind::f16, f32
//                accumulators.  TMEM: Q_A | Q_B | S_A | S_B | O_A | O_B
//                (64+64+64+64+128+128 = 512 columns).  Issue order per tile:
//                PV(A) S'(A) PV(B) S'(B), so one softmax group always has work.
// K and V tiles are double buffered; with Q and P in TMEM the tensor core only
// reads K and V from shared memory.
// The global scales are folded out of the dequantization: s_g(K) goes into the
// softmax scale, s_g(V) into the epilogue.  Both caches compute with f16
// operands (dequantized NVFP4 values are exact there).
// Every mbarrier wait is bounded; on expiry the CTA records NVKV_ERR_TIMEOUT
// in the status word, unwinds, waits for its own MMAs and frees TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "nvkv_internal.h"
#include "ptx.cuh"

namespace nvkv {
namespace {

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

__device__ __forceinline__ uint2 lds8(uint32_t addr)
{
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
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

constexpr int BM = 128;                // rows of one Q tile; a CTA holds two
constexpr int BN = 64;                 // keys per tile
constexpr int NTHREADS = 512;
constexpr int NSTAGE = 4;              // staging ring depth
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait
constexpr int PAIRS_F = 22, PAIRS_H = 21, PAIRS_W = 21;   // 44 / 42 / 42 channels

constexpr uint32_t KV_TILE = 16384;     // 64 keys x 128 x f16
constexpr uint32_t KV_HALF = 8192;      // one 64-element half of a K/V tile
constexpr uint32_t OFF_K = 0;                         // two buffers
constexpr uint32_t OFF_V = OFF_K + 2 * KV_TILE;       // two buffers
constexpr uint32_t OFF_STG = OFF_V + 2 * KV_TILE;     // staging ring
constexpr uint32_t STG_KC = 0, STG_VC = 4096, STG_KS = 8192, STG_VS = 8704;
constexpr uint32_t STG_BYTES = 9216;
constexpr uint32_t OFF_TAB = OFF_STG + NSTAGE * STG_BYTES;   // RoPE tables

// TMEM columns
constexpr uint32_t TM_Q = 0;      // Q_A, Q_B: 64 columns each (f16 pairs)
constexpr uint32_t TM_S = 128;    // S_A, S_B: 64 columns each (f32); P over S
constexpr uint32_t TM_O = 256;    // O_A, O_B: 128 columns each (f32)

enum Bar {
    B_Q = 0,
    B_STG_FULL = 1,                    // + stage
    B_STG_EMPTY = B_STG_FULL + NSTAGE, // + stage
    B_KFULL = B_STG_EMPTY + NSTAGE,    // + buffer
    B_KFREE = B_KFULL + 2,             // + buffer
    B_VFULL = B_KFREE + 2,             // + buffer
    B_VFREE = B_VFULL + 2,             // + buffer
    B_S = B_VFREE + 2,                 // + Q tile: S of that tile written
    B_P = B_S + 2,                     // + Q tile: P of that tile written
    B_ODONE = B_P + 2,
    B_MMADONE = B_ODONE + 1,
    N_BARS = B_MMADONE + 1
};

struct SharedCtl {
    uint64_t bar[N_BARS];
    int abort;
    uint32_t tmem_base;
};

// byte offset of 16-byte chunk c (0..15) of row r inside a 64-row K-major
// operand tile with 128-byte swizzle: two 64-element halves of 8 KB.
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)((c >> 3) * KV_HALF + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 lds16(uint32_t addr)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t lds4(uint32_t addr)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
    return r;
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
    int b, h, q0, n_keys, n_tiles;
    uint32_t sbase;                 // shared-space address of smem
    uint32_t tab_f, tab_h, tab_w;   // byte offsets of the three RoPE tables
};

__device__ __forceinline__ bool wait(Ctx &c, int bar, uint32_t parity)
{
    if (ptx::mbar_wait(&c.ctl->bar[bar], parity, &c.ctl->abort, WAIT_LIMIT_NS)) return true;
    if (atomicExch(&c.ctl->abort, 1) == 0) atomicCAS(c.a->status, 0, (int)NVKV_ERR_TIMEOUT);
    return false;
}

// wait by every lane of a warp, outcome made warp-uniform (the tcgen05 loads
// and stores that follow are warp-collective)
__device__ __forceinline__ bool wait_warp(Ctx &c, int bar, uint32_t parity)
{
    const bool ok = wait(c, bar, parity);
    return __all_sync(0xFFFFFFFFu, ok);
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

__device__ __forceinline__ KeyPos key_pos(const Ctx &c, int key)
{
    const AttnLaunch &a = *c.a;
    KeyPos k;
    k.valid = key < c.n_keys;
    const int kk = k.valid ? key : 0;
    const int f = div_fast(kk, a.T, a.inv_T);
    const int tok = kk - f * a.T;
    const VisFrame vf = a.vis[c.b][f];
    const int hp = div_fast(tok, a.grid_w, a.inv_grid_w);
    k.rr = rope_rows(c, vf.rope_pos, hp, tok - hp * a.grid_w);
    k.grow = (size_t)(c.b * a.H + c.h) * a.R + (size_t)vf.slot * a.T + tok;
    return k;
}

// ------------------------------------------------------------ Q prologue

// Q row `row` of the chunk -> RoPE in f32 -> f16 pairs in TMEM columns
// [tcol, tcol + 64) of this thread's lane.
template <bool FP4>
__device__ void load_q_tmem(const Ctx &c, int row, uint32_t tcol)
{
    const AttnLaunch &a = *c.a;
    const bool valid = row < a.Lq;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.q) +
                       (((size_t)c.b * a.Lq + (valid ? row : 0)) * a.H + c.h) * 16;
    const int frame = valid ? div_fast(row, a.T, a.inv_T) : 0;
    const int tok = valid ? row - frame * a.T : 0;
    const int hp = div_fast(tok, a.grid_w, a.inv_grid_w);
    const RopeRows rr = rope_rows(c, a.q_pos0[c.b] + frame, hp, tok - hp * a.grid_w);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 w = valid ? ldg16(src + hh * 8 + ch) : make_uint4(0, 0, 0, 0);
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int p = hh * 32 + ch * 4 + k;
                const float x = __uint_as_float(u[k] << 16);
                const float y = __uint_as_float(u[k] & 0xFFFF0000u);
                const uint2 e = lds8(rope_at(rr, p));
                float cs, sn;
                if (FP4) {
                    cs = __low2float(as_h2(e.x));
                    sn = __high2float(as_h2(e.y));
                } else {
                    cs = __uint_as_float(e.x);
                    sn = __uint_as_float(e.y);
                }
                o[ch * 4 + k] = pack_f16(x * cs - y * sn, x * sn + y * cs);
            }
        }
        ptx::tmem_st32(tcol + hh * 32, o);
    }
}

// ------------------------------------------------------------ converters

// K, NVFP4: key row r, half HH (channel pairs 32HH .. 32HH+31) from the
// staging stage into the K tile: decode, scale (exact), rotate.  An invalid
// row reads zero codes and writes zeros.
template <int HH>
__device__ __forceinline__ void conv_k_fp4(uint32_t stg, int r, const KeyPos &k, uint32_t kdst)
{
    uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
    uint32_t sc = 0;
    if (k.valid) {
        w0 = lds16(stg + STG_KC + r * 64 + HH * 32);
        w1 = lds16(stg + STG_KC + r * 64 + HH * 32 + 16);
        sc = lds4(stg + STG_KS + r * 8 + HH * 4);
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
        sts16(kdst + swz(r, HH * 8 + cc), o[0], o[1], o[2], o[3]);
    }
}

// V, NVFP4: one key row: decode and scale.
__device__ __forceinline__ void conv_v_fp4(uint32_t stg, int r, bool valid, uint32_t vdst)
{
    uint2 sc = make_uint2(0, 0);
    if (valid) sc = lds8(stg + STG_VS + r * 8);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        const uint4 w = valid ? lds16(stg + STG_VC + r * 64 + g * 16) : make_uint4(0, 0, 0, 0);
        const uint32_t code[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int cc4 = 0; cc4 < 4; ++cc4) {
            const int cc = g * 4 + cc4;                 // output chunk, block cc / 2
            const uint32_t sword = (cc >> 1) < 4 ? sc.x : sc.y;
            const __half2 sb = e4m3_to_h2((sword >> (8 * ((cc >> 1) & 3))) & 0xFFu);
            uint32_t hq[4];
            e2m1x8_to_f16(code[cc4], hq);
            sts16(vdst + swz(r, cc), as_u(__hmul2(as_h2(hq[0]), sb)),
                  as_u(__hmul2(as_h2(hq[1]), sb)), as_u(__hmul2(as_h2(hq[2]), sb)),
                  as_u(__hmul2(as_h2(hq[3]), sb)));
        }
    }
}

// K, bf16 twin: key row r, half HH, read from global memory, RoPE in f32.
template <int HH>
__device__ __forceinline__ void conv_k_bf16(const Ctx &c, int r, const KeyPos &k, uint32_t kdst)
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
        sts16(kdst + swz(r, HH * 8 + cc), o[0], o[1], o[2], o[3]);
    }
}

// V, bf16 twin: one key row from global memory, converted to f16.
__device__ __forceinline__ void conv_v_bf16(const Ctx &c, int r, const KeyPos &k, uint32_t vdst)
{
    const uint4 *src = reinterpret_cast<const uint4 *>(c.a->v_data) + k.grow * 16;
#pragma unroll 4
    for (int cc = 0; cc < 16; ++cc) {
        const uint4 w = k.valid ? ldg16(src + cc) : make_uint4(0, 0, 0, 0);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = pack_f16(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xFFFF0000u));
        sts16(vdst + swz(r, cc), o[0], o[1], o[2], o[3]);
    }
}

// warps 8-11: Q prologue, then K tiles (thread t: key t & 63, half t >> 6)
template <bool FP4>
__device__ void k_converter_role(Ctx &c)
{
    const int t = threadIdx.x - 256;          // 0..127, TMEM lane t
    const uint32_t lane_off = (uint32_t)(t & ~31) << 16;
    const uint32_t tmem = c.ctl->tmem_base;
    load_q_tmem<FP4>(c, c.q0 + t, tmem + lane_off + TM_Q);
    load_q_tmem<FP4>(c, c.q0 + BM + t, tmem + lane_off + TM_Q + 64);
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(&c.ctl->bar[B_Q]);

    const int r = t & 63, hh = t >> 6;        // hh is warp-uniform
    for (int j = 0; j < c.n_tiles; ++j) {
        const int s = j % NSTAGE, kb = j & 1;
        const uint32_t stg = c.sbase + OFF_STG + s * STG_BYTES;
        const uint32_t kdst = c.sbase + OFF_K + kb * KV_TILE;
        const KeyPos k = key_pos(c, j * BN + r);
        if (FP4 && !wait(c, B_STG_FULL + s, (j / NSTAGE) & 1)) return;
        if (j >= 2 && !wait(c, B_KFREE + kb, ((j - 2) >> 1) & 1)) return;
        if (FP4) {
            if (hh == 0) conv_k_fp4<0>(stg, r, k, kdst);
            else conv_k_fp4<1>(stg, r, k, kdst);
        } else {
            if (hh == 0) conv_k_bf16<0>(c, r, k, kdst);
            else conv_k_bf16<1>(c, r, k, kdst);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&c.ctl->bar[B_KFULL + kb]);
        if (FP4) ptx::mbar_arrive(&c.ctl->bar[B_STG_EMPTY + s]);
    }
}

// warps 12-13: V tiles (thread t: key t)
template <bool FP4>
__device__ void v_converter_role(Ctx &c)
{
    const int r = threadIdx.x - 384;          // 0..63
    for (int j = 0; j < c.n_tiles; ++j) {
        const int s = j % NSTAGE, vb = j & 1;
        const uint32_t stg = c.sbase + OFF_STG + s * STG_BYTES;
        const uint32_t vdst = c.sbase + OFF_V + vb * KV_TILE;
        if (FP4 && !wait(c, B_STG_FULL + s, (j / NSTAGE) & 1)) return;
        if (j >= 2 && !wait(c, B_VFREE + vb, ((j - 2) >> 1) & 1)) return;
        if (FP4) {
            conv_v_fp4(stg, r, j * BN + r < c.n_keys, vdst);
        } else {
            const KeyPos k = key_pos(c, j * BN + r);
            conv_v_bf16(c, r, k, vdst);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&c.ctl->bar[B_VFULL + vb]);
        if (FP4) ptx::mbar_arrive(&c.ctl->bar[B_STG_EMPTY + s]);
    }
}

// ------------------------------------------------------------ producer

// Bulk copies of tile j's packed rows: every run of consecutive keys that
// lies in one frame is contiguous in the planes.  Run starts and lengths are
// even (T even), so every copy is 16-byte aligned and sized.
__device__ void producer_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const uint8_t *kc = static_cast<const uint8_t *>(a.k_data);
    const uint8_t *vc = static_cast<const uint8_t *>(a.v_data);
    const uint8_t *ks = static_cast<const uint8_t *>(a.k_scales);
    const uint8_t *vs = static_cast<const uint8_t *>(a.v_scales);
    const size_t head_row0 = (size_t)(c.b * a.H + c.h) * a.R;
    for (int j = 0; j < c.n_tiles; ++j) {
        const int s = j % NSTAGE;
        if (j >= NSTAGE && !wait(c, B_STG_EMPTY + s, ((j - NSTAGE) / NSTAGE) & 1)) return;
        uint8_t *stg = c.smem + OFF_STG + s * STG_BYTES;
        uint64_t *full = &c.ctl->bar[B_STG_FULL + s];
        const int k0 = j * BN;
        const int k1 = min(c.n_keys, k0 + BN);
        ptx::mbar_arrive_expect_tx(full, (uint32_t)(k1 - k0) * 144u);
        for (int k = k0; k < k1;) {
            const int f = div_fast(k, a.T, a.inv_T), tok = k - f * a.T;
            const int n = min(a.T - tok, k1 - k);
            const size_t g = head_row0 + (size_t)a.vis[c.b][f].slot * a.T + tok;
            const int t0 = k - k0;
            ptx::bulk_g2s(stg + STG_KC + t0 * 64, kc + g * 64, (uint32_t)n * 64, full);
            ptx::bulk_g2s(stg + STG_VC + t0 * 64, vc + g * 64, (uint32_t)n * 64, full);
            ptx::bulk_g2s(stg + STG_KS + t0 * 8, ks + g * 8, (uint32_t)n * 8, full);
            ptx::bulk_g2s(stg + STG_VS + t0 * 8, vs + g * 8, (uint32_t)n * 8, full);
            k += n;
        }
    }
}

// ------------------------------------------------------------ MMA issuer

__device__ void mma_role(Ctx &c)
{
    const uint32_t tmem = c.ctl->tmem_base;
    constexpr uint32_t idS = ptx::idesc_f16(kOperandF16, BM, BN, 0);
    constexpr uint32_t idO = ptx::idesc_f16(kOperandF16, BM, 128, 1);
    const uint32_t ks = c.sbase + OFF_K;
    const uint32_t vs = c.sbase + OFF_V;

    // S_tq = Q_tq K^T: A = Q from TMEM (8 x 16 channels), B = K tile, K-major
    auto issue_s = [&](int tq, int kb) {
        const uint32_t kt = ks + kb * KV_TILE;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            ptx::mma_f16_ts(tmem + TM_S + tq * 64, tmem + TM_Q + tq * 64 + kk * 8,
                            ptx::smem_desc_sw128(kt + (kk >> 2) * KV_HALF + (kk & 3) * 32, 16,
                                                 1024),
                            idS, kk > 0);
        ptx::mma_commit(&c.ctl->bar[B_S + tq]);
    };
    // O_tq += P_tq V: A = P from TMEM (4 x 16 keys), B = V tile, MN-major
    auto issue_pv = [&](int tq, int vb, bool first) {
        const uint32_t vt = vs + vb * KV_TILE;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            ptx::mma_f16_ts(tmem + TM_O + tq * 128, tmem + TM_S + tq * 64 + kk * 8,
                            ptx::smem_desc_sw128(vt + kk * 2048, KV_HALF, 1024), idO,
                            (!first || kk > 0) ? 1u : 0u);
    };

    bool ok = wait(c, B_Q, 0) && wait(c, B_KFULL, 0);
    ptx::tc_fence_after();
    if (ok) {
        issue_s(0, 0);
        issue_s(1, 0);
        ptx::mma_commit(&c.ctl->bar[B_KFREE]);
    }
    for (int j = 0; ok && j < c.n_tiles; ++j) {
        const int jn = j + 1, vb = j & 1;
        if (!(ok = wait(c, B_VFULL + vb, (j >> 1) & 1) && wait(c, B_P, j & 1))) break;
        ptx::tc_fence_after();
        issue_pv(0, vb, j == 0);
        if (jn < c.n_tiles) {
            if (!(ok = wait(c, B_KFULL + (jn & 1), (jn >> 1) & 1))) break;
            ptx::tc_fence_after();
            issue_s(0, jn & 1);
        }
        if (!(ok = wait(c, B_P + 1, j & 1))) break;
        ptx::tc_fence_after();
        issue_pv(1, vb, j == 0);
        ptx::mma_commit(&c.ctl->bar[B_VFREE + vb]);
        if (jn < c.n_tiles) {
            issue_s(1, jn & 1);
            ptx::mma_commit(&c.ctl->bar[B_KFREE + (jn & 1)]);
        }
    }
    if (ok) ptx::mma_commit(&c.ctl->bar[B_ODONE]);
    // every MMA this thread issued has finished before TMEM is released
    ptx::mma_commit(&c.ctl->bar[B_MMADONE]);
    const int never = 0;
    ptx::mbar_wait(&c.ctl->bar[B_MMADONE], 0, &never, WAIT_LIMIT_NS);
}

// ------------------------------------------------------------ softmax

template <bool FP4>
__device__ void softmax_role(Ctx &c)
{
    const AttnLaunch &a = *c.a;
    const int warp = threadIdx.x >> 5;
    const int tq = warp >> 2;                       // Q tile A (0) or B (1)
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tmem = c.ctl->tmem_base;
    const uint32_t tS = tmem + TM_S + tq * 64 + lane_off;
    const uint32_t tO = tmem + TM_O + tq * 128 + lane_off;
    const int gi = c.b * a.H + c.h;
    const float sgk = FP4 ? a.s_g[gi] : 1.0f;
    const float sgv = FP4 ? a.s_g[a.B * a.H + gi] : 1.0f;
    const float scale = sgk * 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
    float m = -INFINITY, l = 0.0f;
    for (int j = 0; j < c.n_tiles; ++j) {
        if (!wait_warp(c, B_S + tq, j & 1)) return;
        ptx::tc_fence_after();
        float s[64];
        ptx::tmem_ld32(tS, reinterpret_cast<uint32_t *>(s));
        ptx::tmem_ld32(tS + 32, reinterpret_cast<uint32_t *>(s) + 32);
        ptx::tmem_wait_ld();
        const int nv = c.n_keys - j * BN;
        if (nv < BN) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
                if (i >= nv) s[i] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int i = 1; i < 64; ++i) mx = fmaxf(mx, s[i]);
        const float mt = mx * scale;
        if (__any_sync(0xFFFFFFFFu, mt > m + 8.0f)) {
            const float mn = fmaxf(m, mt);
            const float alpha = ex2(m - mn);     // 0 on the first tile
            l *= alpha;
            m = mn;
            if (j > 0) {
                // PV of the previous tile finished before this tile's S did
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tO + q * 32, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    ptx::tmem_st32(tO + q * 32, o);
                }
            }
        }
        uint32_t pk[32];
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float p0 = ex2(fmaf(s[2 * i], scale, -m));
            const float p1 = ex2(fmaf(s[2 * i + 1], scale, -m));
            sum += p0 + p1;
            pk[i] = pack_f16(p0, p1);
        }
        l += sum;
        ptx::tmem_st32(tS, pk);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.ctl->bar[B_P + tq]);
    }
    if (!wait_warp(c, B_ODONE, 0)) return;
    ptx::tc_fence_after();
    const int row = c.q0 + tq * BM + r;
    const float fin = sgv / l;
    uint4 *dst = reinterpret_cast<uint4 *>(a.out) + (((size_t)c.b * a.Lq + row) * a.H + c.h) * 16;
#pragma unroll 1
    for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        ptx::tmem_ld32(tO + q * 32, o);
        ptx::tmem_wait_ld();
        if (row < a.Lq) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float x = __uint_as_float(o[8 * i + 2 * k]) * fin;
                    const float y = __uint_as_float(o[8 * i + 2 * k + 1]) * fin;
                    __nv_bfloat162 bb = __floats2bfloat162_rn(x, y);
                    w[k] = *reinterpret_cast<uint32_t *>(&bb);
                }
                dst[q * 4 + i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
    }
    if (a.lse && row < a.Lq)
        a.lse[(size_t)(c.b * a.H + c.h) * a.Lq + row] = (m + __log2f(l)) * 0.6931471805599453f;
}

// ------------------------------------------------------------ kernel

template <bool FP4>
__global__ void __launch_bounds__(NTHREADS, 1) k_chunk_attn(const __grid_constant__ AttnLaunch a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctx c;
    c.a = &a;
    c.smem = smem;
    c.sbase = ptx::smem_u32(smem);
    c.b = blockIdx.z;
    c.h = blockIdx.y;
    c.q0 = blockIdx.x * 2 * BM;
    c.n_keys = a.n_vis[c.b] * a.T;
    c.n_tiles = (c.n_keys + BN - 1) / BN;
    c.tab_f = OFF_TAB;
    c.tab_h = c.tab_f + a.n_fpos * PAIRS_F * 8;
    c.tab_w = c.tab_h + a.grid_h * PAIRS_H * 8;
    const uint32_t ctl_off = (c.tab_w + a.grid_w * PAIRS_W * 8 + 63) & ~63u;
    c.ctl = reinterpret_cast<SharedCtl *>(smem + ctl_off);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        // arrival counts: K converters (128) for Q and K full; V converters
        // (64) for V full; both (192) for staging empty; the producer (1, plus
        // bytes) for staging full; tcgen05.commit (1) for what the tensor core
        // signals; a softmax group (128) for P.
        ptx::mbar_init(&c.ctl->bar[B_Q], 128);
        for (int s = 0; s < NSTAGE; ++s) {
            ptx::mbar_init(&c.ctl->bar[B_STG_FULL + s], 1);
            ptx::mbar_init(&c.ctl->bar[B_STG_EMPTY + s], 192);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&c.ctl->bar[B_KFULL + i], 128);
            ptx::mbar_init(&c.ctl->bar[B_KFREE + i], 1);
            ptx::mbar_init(&c.ctl->bar[B_VFULL + i], 64);
            ptx::mbar_init(&c.ctl->bar[B_VFREE + i], 1);
            ptx::mbar_init(&c.ctl->bar[B_S + i], 1);
            ptx::mbar_init(&c.ctl->bar[B_P + i], 128);
        }
        ptx::mbar_init(&c.ctl->bar[B_ODONE], 1);
        ptx::mbar_init(&c.ctl->bar[B_MMADONE], 1);
        c.ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    build_tables<FP4>(c);
    if (warp == 15) {
        ptx::tmem_alloc(&c.ctl->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    if (c.n_tiles > 0) {
        if (warp < 8) {
            softmax_role<FP4>(c);
        } else if (warp < 12) {
            k_converter_role<FP4>(c);
        } else if (warp < 14) {
            v_converter_role<FP4>(c);
        } else if (warp == 14) {
            if (FP4 && (threadIdx.x & 31) == 0) producer_role(c);
        } else if ((threadIdx.x & 31) == 0) {
            mma_role(c);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 15) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(c.ctl->tmem_base, 512);
    }
}

template <bool FP4>
cudaError_t launch(const AttnLaunch &a, cudaStream_t s)
{
    const uint32_t tab =
        (uint32_t)(a.n_fpos * PAIRS_F + a.grid_h * PAIRS_H + a.grid_w * PAIRS_W) * 8;
    const uint32_t bytes = 1024 + OFF_TAB + ((tab + 63) & ~63u) + sizeof(SharedCtl);
    if (bytes > 232448) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(k_chunk_attn<FP4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.Lq + 2 * BM - 1) / (2 * BM), a.H, a.B);
    k_chunk_attn<FP4><<<grid, NTHREADS, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_attention(const AttnLaunch &a, cudaStream_t s)
{
    return a.kv_dtype == NVKV_KV_NVFP4 ? launch<true>(a, s) : launch<false>(a, s);
}

}  // namespace nvkv
