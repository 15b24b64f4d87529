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
// Structure: one CTA per (128 query rows, head, batch); 9 warps.
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r.  Reads S from
//              TMEM, online softmax in registers (lazy rescale of O when the
//              running max grows by more than 2^8), writes P to shared memory.
//   warps 4-7  converters: build the Q operand (RoPE, once), then per tile of
//              128 keys thread r loads key r's packed K/V row, dequantizes
//              (E2M1 -> f16 by cvt, times the E4M3 block scale; exact in f16),
//              rotates K by RoPE in packed f16x2 math and stores both into
//              128-byte-swizzled UMMA operand tiles (double buffered).
//   warp 8     TMEM allocation and the MMA issuer (one thread):
//              S_j = Q K_j^T and O += P_j V_j with tcgen05.mma kind::f16,
//              M = N = 128, accumulators in TMEM (S double buffered, O single).
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

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NTHREADS = 288;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s per wait
constexpr int PAIRS_F = 22, PAIRS_H = 21, PAIRS_W = 21;   // 44 / 42 / 42 channels

constexpr uint32_t TILE_BYTES = 32768;    // 128 rows x 128 x 16-bit
constexpr uint32_t HALF_BYTES = 16384;    // 64-element half of a tile
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE_BYTES;
constexpr uint32_t OFF_V = OFF_K + 2 * TILE_BYTES;
constexpr uint32_t OFF_P = OFF_V + 2 * TILE_BYTES;
constexpr uint32_t OFF_TAB = OFF_P + TILE_BYTES;   // RoPE tables

enum Bar { B_Q = 0, B_KVFULL = 1, B_KVFREE = 3, B_SFULL = 5, B_PFULL = 7, B_ODONE = 8,
           B_MMADONE = 9, N_BARS = 10 };

struct SharedCtl {
    uint64_t bar[N_BARS];
    int abort;
    uint32_t tmem_base;
};

// byte offset of 16-byte chunk c (0..15) of row r inside a 128-row K-major
// operand tile with 128-byte swizzle: two 64-element halves of 16 KB.
__device__ __forceinline__ uint32_t swz(int r, int c)
{
    return (uint32_t)((c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4));
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

__device__ __forceinline__ uint2 ldg8(const void *p)
{
    uint2 r;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ void sts16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                      uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
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

// two E4M3 bytes -> f16x2 (exact)
__device__ __forceinline__ uint32_t e4m3x2_to_f16(uint32_t two_bytes)
{
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)two_bytes));
    return r;
}

__device__ __forceinline__ uint2 lds8(uint32_t addr)
{
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
    return r;
}

__device__ __forceinline__ __half2 as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }
__device__ __forceinline__ uint32_t as_u(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

// RoPE table entry.  NVFP4 path: (c, c) and (-s, s) as f16x2; bf16 twin: (c, s) f32.
struct RopeH { uint32_t cc, ns; };

// Both caches feed the tensor cores f16 operands (kind::f16, f32 accumulate).
// NVFP4: code * s_b is exact in f16.  bf16 twin: cached values convert to f16
// exactly inside f16's normal range (|x| in [2^-14, 65504]); rotated keys,
// queries and probabilities keep 3 more mantissa bits than bf16 would.
constexpr uint32_t kOperandF16 = 0;

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi)
{
    return as_u(__floats2half2_rn(lo, hi));
}

struct Ctx {
    const AttnLaunch *a;
    uint8_t *smem;
    SharedCtl *ctl;
    int b, h, q0, n_keys, n_tiles;
    uint32_t tab_f, tab_h, tab_w;   // smem byte offsets of the three RoPE tables
    uint32_t sbase;                 // shared-space address of smem
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

// smem byte offset of the table entry for channel pair p of a token at
// (frame position fpos, row hp, column wp)
__device__ __forceinline__ uint32_t rope_entry(const Ctx &c, int p, int fpos, int hp, int wp)
{
    if (p < PAIRS_F) return c.tab_f + (fpos * PAIRS_F + p) * 8;
    if (p < PAIRS_F + PAIRS_H) return c.tab_h + (hp * PAIRS_H + (p - PAIRS_F)) * 8;
    return c.tab_w + (wp * PAIRS_W + (p - PAIRS_F - PAIRS_H)) * 8;
}

__device__ __forceinline__ void rope_cs_f32(const Ctx &c, bool fp4, uint32_t off, float &cs,
                                            float &sn)
{
    const uint2 e = lds8(c.sbase + off);
    if (fp4) {
        cs = __low2float(as_h2(e.x));
        sn = __high2float(as_h2(e.y));
    } else {
        cs = __uint_as_float(e.x);
        sn = __uint_as_float(e.y);
    }
}

// ------------------------------------------------------------ converters

template <bool FP4>
__device__ void load_q(Ctx &c, int r)
{
    const AttnLaunch &a = *c.a;
    const int row = c.q0 + r;
    const uint32_t qs = ptx::smem_u32(c.smem + OFF_Q);
    uint4 w[16];
    if (row < a.Lq) {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.q) +
                           (((size_t)c.b * a.Lq + row) * a.H + c.h) * 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = ldg16(src + i);
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = make_uint4(0, 0, 0, 0);
    }
    const int frame = row < a.Lq ? row / a.T : 0;
    const int tok = row < a.Lq ? row - frame * a.T : 0;
    const int fpos = a.q_pos0[c.b] + frame, hp = tok / a.grid_w, wp = tok - hp * a.grid_w;
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {
        const uint32_t u[4] = {w[ch].x, w[ch].y, w[ch].z, w[ch].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int p = ch * 4 + k;
            const float x = __uint_as_float(u[k] << 16), y = __uint_as_float(u[k] & 0xFFFF0000u);
            float cs, sn;
            rope_cs_f32(c, FP4, rope_entry(c, p, fpos, hp, wp), cs, sn);
            o[k] = pack_f16(x * cs - y * sn, x * sn + y * cs);
        }
        sts16(qs + swz(r, ch), o[0], o[1], o[2], o[3]);
    }
}

struct KeyRow {
    int valid, fpos, hp, wp;
    size_t row;   // global row index into the [B][H][R] planes
};

__device__ __forceinline__ KeyRow key_row(const Ctx &c, int j, int r)
{
    const AttnLaunch &a = *c.a;
    KeyRow k;
    const int key = j * BN + r;
    k.valid = key < c.n_keys;
    const int kk = k.valid ? key : 0;
    const int f = kk / a.T, tok = kk - f * a.T;
    const VisFrame vf = a.vis[c.b][f];
    k.fpos = vf.rope_pos;
    k.hp = tok / a.grid_w;
    k.wp = tok - k.hp * a.grid_w;
    k.row = (size_t)(c.b * a.H + c.h) * a.R + (size_t)vf.slot * a.T + tok;
    return k;
}

struct Fp4Row { uint4 kc[4], vc[4]; uint2 ks, vs; };

__device__ __forceinline__ void load_fp4_row(const Ctx &c, const KeyRow &k, Fp4Row &d)
{
    const AttnLaunch &a = *c.a;
    if (!k.valid) {
#pragma unroll
        for (int i = 0; i < 4; ++i) d.kc[i] = d.vc[i] = make_uint4(0, 0, 0, 0);
        d.ks = d.vs = make_uint2(0, 0);
        return;
    }
    const uint8_t *kc = static_cast<const uint8_t *>(a.k_data) + k.row * 64;
    const uint8_t *vc = static_cast<const uint8_t *>(a.v_data) + k.row * 64;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        d.kc[i] = ldg16(kc + 16 * i);
        d.vc[i] = ldg16(vc + 16 * i);
    }
    d.ks = ldg8(static_cast<const uint8_t *>(a.k_scales) + k.row * 8);
    d.vs = ldg8(static_cast<const uint8_t *>(a.v_scales) + k.row * 8);
}

// f16x2 (s_b, s_b) of block `blk` from the row's eight scale bytes
__device__ __forceinline__ __half2 block_scale(uint2 s, int blk)
{
    const uint32_t w = blk < 4 ? s.x : s.y;
    const uint32_t two = (w >> (((blk & 3) >> 1) * 16)) & 0xFFFFu;
    const __half2 pair = as_h2(e4m3x2_to_f16(two));
    return (blk & 1) ? __high2half2(pair) : __low2half2(pair);
}

__device__ void convert_fp4_row(const Ctx &c, int r, const KeyRow &k, const Fp4Row &d,
                                uint32_t kdst, uint32_t vdst)
{
#pragma unroll
    for (int ch = 0; ch < 16; ++ch) {        // 16-byte output chunk = 4 pairs
        const uint4 kw = d.kc[ch >> 2];
        const uint4 vw = d.vc[ch >> 2];
        const uint32_t kword = (ch & 3) == 0 ? kw.x : (ch & 3) == 1 ? kw.y : (ch & 3) == 2 ? kw.z : kw.w;
        const uint32_t vword = (ch & 3) == 0 ? vw.x : (ch & 3) == 1 ? vw.y : (ch & 3) == 2 ? vw.z : vw.w;
        const __half2 ksb = block_scale(d.ks, ch >> 1);
        const __half2 vsb = block_scale(d.vs, ch >> 1);
        uint32_t kh[4], vh[4], ko[4], vo[4];
        e2m1x8_to_f16(kword, kh);
        e2m1x8_to_f16(vword, vh);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = ch * 4 + q;
            const __half2 kv = __hmul2(as_h2(kh[q]), ksb);     // (x, y) * s_b, exact
            const uint2 e = lds8(c.sbase + rope_entry(c, p, k.fpos, k.hp, k.wp));
            // (x c - y s, y c + x s)
            const __half2 rot = __hfma2(__lowhigh2highlow(kv), as_h2(e.y), __hmul2(kv, as_h2(e.x)));
            ko[q] = as_u(rot);
            vo[q] = as_u(__hmul2(as_h2(vh[q]), vsb));
        }
        sts16(kdst + swz(r, ch), ko[0], ko[1], ko[2], ko[3]);
        sts16(vdst + swz(r, ch), vo[0], vo[1], vo[2], vo[3]);
    }
}

__device__ void convert_bf16_row(const Ctx &c, int r, const KeyRow &k, uint32_t kdst,
                                 uint32_t vdst)
{
    const AttnLaunch &a = *c.a;
    const uint4 *ks = reinterpret_cast<const uint4 *>(a.k_data) + k.row * 16;
    const uint4 *vs = reinterpret_cast<const uint4 *>(a.v_data) + k.row * 16;
#pragma unroll 4
    for (int ch = 0; ch < 16; ++ch) {
        const uint4 kw = k.valid ? ldg16(ks + ch) : make_uint4(0, 0, 0, 0);
        const uint4 vw = k.valid ? ldg16(vs + ch) : make_uint4(0, 0, 0, 0);
        const uint32_t u[4] = {kw.x, kw.y, kw.z, kw.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int p = ch * 4 + q;
            const float x = __uint_as_float(u[q] << 16), y = __uint_as_float(u[q] & 0xFFFF0000u);
            float cs, sn;
            rope_cs_f32(c, false, rope_entry(c, p, k.fpos, k.hp, k.wp), cs, sn);
            o[q] = pack_f16(x * cs - y * sn, x * sn + y * cs);
        }
        const uint32_t vu[4] = {vw.x, vw.y, vw.z, vw.w};
        uint32_t vo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            vo[q] = pack_f16(__uint_as_float(vu[q] << 16), __uint_as_float(vu[q] & 0xFFFF0000u));
        sts16(kdst + swz(r, ch), o[0], o[1], o[2], o[3]);
        sts16(vdst + swz(r, ch), vo[0], vo[1], vo[2], vo[3]);
    }
}

template <bool FP4>
__device__ void converter_role(Ctx &c)
{
    const int r = threadIdx.x - 128;
    load_q<FP4>(c, r);
    ptx::fence_proxy_async_smem();
    ptx::mbar_arrive(&c.ctl->bar[B_Q]);

    const uint32_t kbase = ptx::smem_u32(c.smem + OFF_K);
    const uint32_t vbase = ptx::smem_u32(c.smem + OFF_V);
    KeyRow kr = key_row(c, 0, r);
    Fp4Row cur, nxt;
    if (FP4) load_fp4_row(c, kr, cur);
    for (int j = 0; j < c.n_tiles; ++j) {
        KeyRow kn = kr;
        if (FP4 && j + 1 < c.n_tiles) {
            kn = key_row(c, j + 1, r);
            load_fp4_row(c, kn, nxt);
        }
        if (j >= 2 && !wait(c, B_KVFREE + (j & 1), ((j - 2) >> 1) & 1)) return;
        const uint32_t kd = kbase + (j & 1) * TILE_BYTES, vd = vbase + (j & 1) * TILE_BYTES;
        if (FP4) {
            convert_fp4_row(c, r, kr, cur, kd, vd);
        } else {
            convert_bf16_row(c, r, kr, kd, vd);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&c.ctl->bar[B_KVFULL + (j & 1)]);
        if (FP4) {
            cur = nxt;
            kr = kn;
        } else if (j + 1 < c.n_tiles) {
            kr = key_row(c, j + 1, r);
        }
    }
}

// ------------------------------------------------------------ MMA issuer

template <bool FP4>
__device__ void mma_role(Ctx &c)
{
    const uint32_t tmem = c.ctl->tmem_base;
    const uint32_t tS[2] = {tmem, tmem + 128};
    const uint32_t tO = tmem + 256;
    constexpr uint32_t idS = ptx::idesc_f16(kOperandF16, BM, BN, 0);
    constexpr uint32_t idO = ptx::idesc_f16(kOperandF16, BM, 128, 1);
    const uint32_t qs = ptx::smem_u32(c.smem + OFF_Q);
    const uint32_t ks = ptx::smem_u32(c.smem + OFF_K);
    const uint32_t vs = ptx::smem_u32(c.smem + OFF_V);
    const uint32_t ps = ptx::smem_u32(c.smem + OFF_P);
    bool ok = wait(c, B_Q, 0);
    ptx::tc_fence_after();
    for (int j = -1; ok && j < c.n_tiles; ++j) {
        const int jn = j + 1;
        if (jn < c.n_tiles) {
            if (!(ok = wait(c, B_KVFULL + (jn & 1), (jn >> 1) & 1))) break;
            ptx::tc_fence_after();
            const uint32_t kt = ks + (jn & 1) * TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                ptx::mma_f16_ss(tS[jn & 1], ptx::smem_desc_sw128(qs + off, 16, 1024),
                                ptx::smem_desc_sw128(kt + off, 16, 1024), idS, kk > 0);
            }
            ptx::mma_commit(&c.ctl->bar[B_SFULL + (jn & 1)]);
        }
        if (j >= 0) {
            if (!(ok = wait(c, B_PFULL, j & 1))) break;
            ptx::tc_fence_after();
            const uint32_t vt = vs + (j & 1) * TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t aoff = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                ptx::mma_f16_ss(tO, ptx::smem_desc_sw128(ps + aoff, 16, 1024),
                                ptx::smem_desc_sw128(vt + kk * 2048, HALF_BYTES, 1024), idO,
                                (j > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(&c.ctl->bar[B_ODONE]);
            ptx::mma_commit(&c.ctl->bar[B_KVFREE + (j & 1)]);
        }
    }
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
    const int r = threadIdx.x;
    const int warp = r >> 5;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tmem = c.ctl->tmem_base;
    const uint32_t tS[2] = {tmem + lane_off, tmem + 128 + lane_off};
    const uint32_t tO = tmem + 256 + lane_off;
    const uint32_t ps = ptx::smem_u32(c.smem + OFF_P);
    const int gi = c.b * a.H + c.h;
    const float sgk = FP4 ? a.s_g[gi] : 1.0f;
    const float sgv = FP4 ? a.s_g[a.B * a.H + gi] : 1.0f;
    const float scale = sgk * 1.4426950408889634f * 0.08838834764831845f;   // log2(e)/sqrt(128)
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < c.n_tiles; ++j) {
        if (!(ok = wait_warp(c, B_SFULL + (j & 1), (j >> 1) & 1))) break;
        ptx::tc_fence_after();
        float s[128];
#pragma unroll
        for (int q = 0; q < 4; ++q) ptx::tmem_ld32(tS[j & 1] + q * 32, reinterpret_cast<uint32_t *>(s) + q * 32);
        ptx::tmem_wait_ld();
        const int nv = min(BN, c.n_keys - j * BN);
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i)
            if (i < nv) mx = fmaxf(mx, s[i]);
        const float mt = mx * scale;
        const bool need = __any_sync(0xFFFFFFFFu, mt > m + 8.0f);
        if (need) {
            const float mn = fmaxf(m, mt);
            const float alpha = ex2(m - mn);     // 0 on the first tile
            l *= alpha;
            m = mn;
            if (j > 0) {
                if (!(ok = wait_warp(c, B_ODONE, (j - 1) & 1))) break;
                ptx::tc_fence_after();
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t o[32];
                    ptx::tmem_ld32(tO + q * 32, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    ptx::tmem_st32(tO + q * 32, o);
                }
                ptx::tmem_wait_st();
            }
        }
        uint32_t pk[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const float p0 = (2 * i < nv) ? ex2(s[2 * i] * scale - m) : 0.0f;
            const float p1 = (2 * i + 1 < nv) ? ex2(s[2 * i + 1] * scale - m) : 0.0f;
            l += p0 + p1;
            pk[i] = pack_f16(p0, p1);
        }
        if (j > 0 && !(ok = wait_warp(c, B_ODONE, (j - 1) & 1))) break;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch)
            sts16(ps + swz(r, ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.ctl->bar[B_PFULL]);
    }
    if (!ok) return;
    if (!wait_warp(c, B_ODONE, (c.n_tiles - 1) & 1)) return;
    ptx::tc_fence_after();
    const int row = c.q0 + r;
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
    c.q0 = blockIdx.x * BM;
    c.n_keys = a.n_vis[c.b] * a.T;
    c.n_tiles = (c.n_keys + BN - 1) / BN;
    c.tab_f = OFF_TAB;
    c.tab_h = c.tab_f + a.n_fpos * PAIRS_F * 8;
    c.tab_w = c.tab_h + a.grid_h * PAIRS_H * 8;
    const uint32_t ctl_off = (c.tab_w + a.grid_w * PAIRS_W * 8 + 63) & ~63u;
    c.ctl = reinterpret_cast<SharedCtl *>(smem + ctl_off);
    const int warp = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        ptx::mbar_init(&c.ctl->bar[B_Q], 128);
        ptx::mbar_init(&c.ctl->bar[B_KVFULL], 128);
        ptx::mbar_init(&c.ctl->bar[B_KVFULL + 1], 128);
        ptx::mbar_init(&c.ctl->bar[B_KVFREE], 1);
        ptx::mbar_init(&c.ctl->bar[B_KVFREE + 1], 1);
        ptx::mbar_init(&c.ctl->bar[B_SFULL], 1);
        ptx::mbar_init(&c.ctl->bar[B_SFULL + 1], 1);
        ptx::mbar_init(&c.ctl->bar[B_PFULL], 128);
        ptx::mbar_init(&c.ctl->bar[B_ODONE], 1);
        ptx::mbar_init(&c.ctl->bar[B_MMADONE], 1);
        c.ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    build_tables<FP4>(c);
    if (warp == 8) {
        ptx::tmem_alloc(&c.ctl->tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();

    if (c.n_tiles > 0) {
        if (warp < 4) {
            softmax_role<FP4>(c);
        } else if (warp < 8) {
            converter_role<FP4>(c);
        } else if ((threadIdx.x & 31) == 0) {
            mma_role<FP4>(c);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(c.ctl->tmem_base, 512);
    }
}

template <bool FP4>
cudaError_t launch(const AttnLaunch &a, cudaStream_t s)
{
    const uint32_t tab = (uint32_t)(a.n_fpos * PAIRS_F + a.grid_h * PAIRS_H + a.grid_w * PAIRS_W) * 8;
    const uint32_t bytes = 1024 + OFF_TAB + ((tab + 63) & ~63u) + sizeof(SharedCtl);
    if (bytes > 232448) return cudaErrorInvalidConfiguration;
    cudaError_t e = cudaFuncSetAttribute(k_chunk_attn<FP4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((a.Lq + BM - 1) / BM, a.H, a.B);
    k_chunk_attn<FP4><<<grid, NTHREADS, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_attention(const AttnLaunch &a, cudaStream_t s)
{
    return a.kv_dtype == NVKV_KV_NVFP4 ? launch<true>(a, s) : launch<false>(a, s);
}

}  // namespace nvkv
