// K/V projection of one chunk on tcgen05 with the NVFP4 append fused into
// its epilogue (sm_100a).
//
// K = x W_k^T and V = x W_v^T for the chunk's hidden states x [B*Lq][hidden]
// and weights W [H*128][hidden] (bf16 in, f32 accumulate), then, per
// token-head row of 128 channels, rounding to bf16 (the projection's output
// type) and either storing it (mode 0) or quantizing it to NVFP4 straight
// into the row's ring slot (mode 1: in-place quantized KV-cache update,
// "NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
// generation", section "NVFP4, sequence parallel and the async decode path";
// the bf16 K/V never reaches HBM).
//
// Structure: a cluster of two CTAs (one per SM) computes a 256 x 256 output
// tile: 256 token rows (128 per CTA) by the 128 channels of each of two
// heads (of K, of V, or one of each).  Every MMA is a pair MMA (cta_group::2,
// M = 256, N = 256, both operands in shared memory, 128-byte swizzle), issued
// by the even CTA; per 64-element step of hidden each CTA stages, by TMA, its
// own 128 rows of x and the 128 weight rows of its head of the pair (B is
// split along N between the two CTAs), in a 6-stage ring.  Against 256 x 128
// tiles this cuts the operand traffic from L2 per FLOP by a third, which is
// what bounds the kernel.  The accumulator (256 columns) is double buffered
// in TMEM so that the epilogue of one tile overlaps the MMAs of the next.
// Warps:
//   warp 0       producer (TMA) in both CTAs
//   warp 1       TMEM allocation; MMA issuer (even CTA) or relay of the
//                stage-full events (odd CTA)
//   warp 2       odd CTA: relay of the accumulator-free events
//   warps 4-7    epilogue: thread r owns output row r of the CTA's half
// The grid is persistent; tiles run M-tile-major so that concurrent pairs
// share x rows in L2.  Every wait is bounded; on expiry the pair records
// NVKV_ERR_TIMEOUT in the status word and unwinds.
#include <cuda.h>
#include <cuda_bf16.h>

#include "nvfp4_quant.cuh"
#include "nvkv_internal.h"
#include "ptx.cuh"

namespace nvkv {
namespace {

constexpr int PM = 128;                            // rows per CTA
constexpr int PK = 64;                             // hidden elements per stage
constexpr int NST = 6;                             // stages
constexpr uint32_t A_BYTES = PM * PK * 2;          // 16 KB
constexpr uint32_t B_BYTES = 128 * PK * 2;         // 16 KB: one head's 128 channels
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int PTHREADS = 256;
constexpr uint64_t PWAIT_NS = 2000000000ull;       // 2 s per wait

enum PBar {
    P_FULL = 0,                    // + stage: this CTA's TMA bytes landed
    P_PFULL = P_FULL + NST,        // + stage: [even] the odd CTA's stage landed (relay)
    P_EMPTY = P_PFULL + NST,       // + stage: the stage's MMAs are done (commit)
    P_AFULL = P_EMPTY + NST,       // + buffer: accumulator complete (commit)
    P_AEMPTY = P_AFULL + 2,        // + buffer: epilogue read it (128, + relay in the even CTA)
    P_DONE = P_AEMPTY + 2,         // every MMA issued is done (commit)
    P_NBARS = P_DONE + 1
};

struct PCtl {
    uint64_t bar[P_NBARS];
    int abort;
    uint32_t tmem_base;
};

struct PCtx {
    const ProjLaunch *p;
    PCtl *ctl;
    uint8_t *stages;
    uint32_t rank;
    uint32_t lead_bar;             // shared::cluster address of the even CTA's bar[0]
    uint32_t peer_abort;
    int n_tiles, nk, pair;
    int n_full, n_items;           // tiles in whole waves; work items (see item_of)
};

// Work item v of the persistent schedule.  Tiles are 256 x 256 (two heads);
// when the tiles left after the last whole wave fit twice into one wave,
// each of them runs as two 256 x 128 halves (one head each, N = 128 MMAs) on
// two pairs, which halves that wave's length.  half = -1: the whole tile.
struct Item {
    int t, half;
};

__device__ __forceinline__ Item item_of(const PCtx &c, int v)
{
    if (v < c.n_full) return {v, -1};
    const int h = v - c.n_full;
    return {c.n_full + (h >> 1), h & 1};
}

__device__ __forceinline__ void pset_abort(PCtx &c)
{
    if (atomicExch(&c.ctl->abort, 1) == 0) {
        atomicCAS(c.p->status, 0, (int)NVKV_ERR_TIMEOUT);
        ptx::st_cluster_u32(c.peer_abort, 1u);
    }
}

__device__ __forceinline__ bool pwait(PCtx &c, int bar, uint32_t parity)
{
    if (ptx::mbar_wait(&c.ctl->bar[bar], parity, &c.ctl->abort, PWAIT_NS)) return true;
    pset_abort(c);
    return false;
}

__device__ __forceinline__ bool pwait_warp(PCtx &c, int bar, uint32_t parity)
{
    const bool ok = pwait(c, bar, parity);
    return __all_sync(0xFFFFFFFFu, ok);
}

__device__ void producer(PCtx &c, const CUtensorMap *tx, const CUtensorMap *twk,
                         const CUtensorMap *twv)
{
    const ProjLaunch &p = *c.p;
    ptx::prefetch_tensormap(tx);
    ptx::prefetch_tensormap(twk);
    ptx::prefetch_tensormap(twv);
    int it = 0;
    bool ok = true;
    for (int v = c.pair; ok && v < c.n_items; v += p.n_pairs) {
        const Item w = item_of(c, v);
        const int mt = w.t / p.H, tt = w.t - mt * p.H;
        // whole tile: this CTA's head of the pair; half tile: this CTA's 64
        // rows of the one head (the box's other 64 rows go unused)
        const int hh = 2 * tt + (w.half < 0 ? (int)c.rank : w.half);
        const CUtensorMap *tw = hh < p.H ? twk : twv;
        const int wrow = (hh < p.H ? hh : hh - p.H) * 128 + (w.half < 0 ? 0 : 64 * (int)c.rank);
        const int xrow = mt * 2 * PM + PM * (int)c.rank;
        for (int ks = 0; ks < c.nk; ++ks, ++it) {
            const int s = it % NST;
            if (it >= NST && !(ok = pwait(c, P_EMPTY + s, (it / NST - 1) & 1))) break;
            uint8_t *st = c.stages + s * STAGE_BYTES;
            uint64_t *full = &c.ctl->bar[P_FULL + s];
            ptx::mbar_arrive_expect_tx(full, STAGE_BYTES);
            ptx::tma_load_2d(st, tx, ks * PK, xrow, full);
            ptx::tma_load_2d(st + A_BYTES, tw, ks * PK, wrow, full);
        }
    }
    // no CTA leaves with copies into its shared memory in flight
    const int never = 0;
    for (int i = it - 1; i >= 0 && i >= it - NST; --i)
        ptx::mbar_wait(&c.ctl->bar[P_FULL + i % NST], (i / NST) & 1, &never, PWAIT_NS);
}

__device__ void mma_issuer(PCtx &c)
{
    const ProjLaunch &p = *c.p;
    const uint32_t tmem = c.ctl->tmem_base;
    constexpr uint32_t idesc256 = ptx::idesc_f16(1 /* bf16 */, 2 * PM, 256, 0);
    constexpr uint32_t idesc128 = ptx::idesc_f16(1 /* bf16 */, 2 * PM, 128, 0);
    const uint16_t both = 0x3;
    int it = 0, j = 0;
    bool ok = true;
    for (int v = c.pair; ok && v < c.n_items; v += p.n_pairs, ++j) {
        const uint32_t idesc = item_of(c, v).half < 0 ? idesc256 : idesc128;
        const int b = j & 1;
        if (j >= 2 && !(ok = pwait(c, P_AEMPTY + b, ((j - 2) >> 1) & 1))) break;
        ptx::tc_fence_after();
        for (int ks = 0; ks < c.nk; ++ks, ++it) {
            const int s = it % NST;
            const uint32_t par = (it / NST) & 1;
            if (!(ok = pwait(c, P_FULL + s, par) && pwait(c, P_PFULL + s, par))) break;
            ptx::tc_fence_after();
            const uint32_t a0 = ptx::smem_u32(c.stages + s * STAGE_BYTES), b0 = a0 + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < PK / 16; ++kk)
                ptx::mma2_f16_ss(tmem + b * 256, ptx::smem_desc_sw128(a0 + kk * 32, 16, 1024),
                                 ptx::smem_desc_sw128(b0 + kk * 32, 16, 1024), idesc,
                                 (ks | kk) ? 1u : 0u);
            ptx::mma2_commit_mc(&c.ctl->bar[P_EMPTY + s], both);
        }
        if (!ok) break;
        ptx::mma2_commit_mc(&c.ctl->bar[P_AFULL + b], both);
    }
    ptx::mma2_commit_mc(&c.ctl->bar[P_DONE], both);
}

// odd CTA: forward each stage-full phase to the even CTA's P_PFULL
__device__ void relay_full(PCtx &c)
{
    const ProjLaunch &p = *c.p;
    int it = 0;
    for (int v = c.pair; v < c.n_items; v += p.n_pairs)
        for (int ks = 0; ks < c.nk; ++ks, ++it) {
            const int s = it % NST;
            if (!pwait(c, P_FULL + s, (it / NST) & 1)) return;
            ptx::mbar_arrive_remote(c.lead_bar + (P_PFULL + s) * 8);
        }
}

// odd CTA: forward each accumulator-free phase to the even CTA's P_AEMPTY
__device__ void relay_aempty(PCtx &c)
{
    const ProjLaunch &p = *c.p;
    int j = 0;
    for (int v = c.pair; v < c.n_items; v += p.n_pairs, ++j) {
        const int b = j & 1;
        if (!pwait(c, P_AEMPTY + b, (j >> 1) & 1)) return;
        ptx::mbar_arrive_remote(c.lead_bar + (P_AEMPTY + b) * 8);
    }
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ void epilogue(PCtx &c)
{
    const ProjLaunch &p = *c.p;
    const int r = threadIdx.x - 128;                   // TMEM lane = row of the CTA's half
    const uint32_t tbase = c.ctl->tmem_base + ((uint32_t)(r & ~31) << 16);
    int j = 0;
    for (int v = c.pair; v < c.n_items; v += p.n_pairs, ++j) {
        const int b = j & 1;
        if (!pwait_warp(c, P_AFULL + b, (j >> 1) & 1)) return;
        ptx::tc_fence_after();
        const Item wi = item_of(c, v);
        const int t = wi.t, mt = t / p.H;
        const int row = mt * 2 * PM + PM * (int)c.rank + r;
        const bool valid = row < p.M;
        const int bi = valid ? row / p.Lq : 0, l = valid ? row - bi * p.Lq : 0;
        int frame = 0, tok = 0;
        if (p.mode == 1) {
            frame = l / p.T;
            tok = l - frame * p.T;
        }
        const int h0 = wi.half < 0 ? 0 : wi.half, h1 = wi.half < 0 ? 2 : wi.half + 1;
#pragma unroll 1
        for (int hs = h0; hs < h1; ++hs) {
            // head of accumulator columns [128 col, +128): the tile's two
            // heads in turn, or the half tile's one head in columns 0-127
            const int hh = 2 * (t - mt * p.H) + hs;
            const int col = wi.half < 0 ? hs : 0;
            const int kv = hh < p.H ? 0 : 1, h = hh - kv * p.H;
            size_t drow = 0;
            float sg = 1.0f;
            if (p.mode == 1) {
                drow = (size_t)(bi * p.H + h) * p.R + (size_t)p.slot[bi * p.C + frame] * p.Tr + tok;
                sg = p.s_g[(kv * p.B + bi) * p.H + h];
            }
#pragma unroll 1
            for (int q = 0; q < 4; ++q) {
                uint32_t d[32];
                ptx::tmem_ld32(tbase + b * 256 + col * 128 + q * 32, d);
                ptx::tmem_wait_ld();
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = bf16x2_bits(__uint_as_float(d[2 * i]), __uint_as_float(d[2 * i + 1]));
                if (!valid) continue;
                if (p.mode == 0) {
                    uint4 *dst = reinterpret_cast<uint4 *>(kv ? p.v_out : p.k_out) +
                                 (((size_t)bi * p.Lq + l) * p.H + h) * 16 + q * 4;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                } else {
                    uint2 c0, c1;
                    const uint32_t s0 = q4::quantize_block(make_uint4(w[0], w[1], w[2], w[3]),
                                                           make_uint4(w[4], w[5], w[6], w[7]), sg, c0);
                    const uint32_t s1 = q4::quantize_block(make_uint4(w[8], w[9], w[10], w[11]),
                                                           make_uint4(w[12], w[13], w[14], w[15]), sg,
                                                           c1);
                    *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(kv ? p.v_data : p.k_data) +
                                               drow * 64 + q * 16) = make_uint4(c0.x, c0.y, c1.x, c1.y);
                    *reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(kv ? p.v_scales : p.k_scales) +
                                                  drow * 8 + q * 2) = (uint16_t)(s0 | (s1 << 8));
                }
            }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&c.ctl->bar[P_AEMPTY + b]);
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PTHREADS, 1)
    k_kv_project(const __grid_constant__ ProjLaunch p, const __grid_constant__ CUtensorMap tx,
                 const __grid_constant__ CUtensorMap twk, const __grid_constant__ CUtensorMap twv)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PCtx c;
    c.p = &p;
    c.stages = smem;
    c.ctl = reinterpret_cast<PCtl *>(smem + NST * STAGE_BYTES);
    c.rank = ptx::cluster_ctarank();
    c.pair = blockIdx.x >> 1;
    c.nk = p.hidden / PK;
    c.n_tiles = (p.M + 2 * PM - 1) / (2 * PM) * p.H;
    c.n_full = c.n_tiles / p.n_pairs * p.n_pairs;
    c.n_items = 2 * (c.n_tiles - c.n_full) <= p.n_pairs ? c.n_full + 2 * (c.n_tiles - c.n_full)
                                                        : c.n_tiles;
    if (c.n_items == c.n_tiles) c.n_full = c.n_tiles;
    c.lead_bar = ptx::mapa(ptx::smem_u32(&c.ctl->bar[0]), 0);
    c.peer_abort = ptx::mapa(ptx::smem_u32(&c.ctl->abort), c.rank ^ 1u);
    const int warp = threadIdx.x >> 5;
    const bool lane0 = (threadIdx.x & 31) == 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < P_NBARS; ++i) {
            uint32_t n = 1;
            if (i == P_AEMPTY || i == P_AEMPTY + 1) n = c.rank == 0 ? 129 : 128;
            ptx::mbar_init(&c.ctl->bar[i], n);
        }
        c.ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc2(&c.ctl->tmem_base, 512);
        ptx::tmem_relinquish2();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();          // peer barriers initialised before any remote arrive
    ptx::tc_fence_after();

    if (warp == 0) {
        if (lane0) producer(c, &tx, &twk, &twv);
    } else if (warp == 1) {
        if (lane0) {
            if (c.rank == 0) mma_issuer(c);
            else relay_full(c);
        }
        __syncwarp();
        // both CTAs: every MMA touching this CTA's TMEM or shared memory is done
        const int never = 0;
        if (lane0) ptx::mbar_wait(&c.ctl->bar[P_DONE], 0, &never, PWAIT_NS);
        __syncwarp();
    } else if (warp == 2) {
        if (lane0 && c.rank == 1) relay_aempty(c);
    } else if (warp >= 4) {
        epilogue(c);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();          // no CTA leaves while its peer may touch its memory
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc2(c.ctl->tmem_base, 512);
    }
}

typedef CUresult (*EncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn()
{
    static EncodeTiled fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(f);
    }
    return fn;
}

// bf16 [rows][cols] row-major, boxes of box_rows x 64 elements, 128-byte swizzle;
// rows past the end read as zeros
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiled fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)PK, box_rows};
    const cuuint32_t elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_kv_project(const ProjLaunch &p_in, const void *x, const void *w_k,
                              const void *w_v, cudaStream_t s)
{
    ProjLaunch p = p_in;
    CUtensorMap tx, twk, twv;
    if (!make_map(&tx, x, (uint64_t)p.M, (uint64_t)p.hidden, PM) ||
        !make_map(&twk, w_k, (uint64_t)p.H * 128, (uint64_t)p.hidden, 128) ||
        !make_map(&twv, w_v, (uint64_t)p.H * 128, (uint64_t)p.hidden, 128))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int n_tiles = (p.M + 2 * PM - 1) / (2 * PM) * p.H;
    p.n_pairs = sms / 2 < n_tiles ? sms / 2 : n_tiles;
    if (p.n_pairs < 1) return cudaErrorInvalidConfiguration;
    const int bytes = 1024 + NST * STAGE_BYTES + (int)sizeof(PCtl);
    e = cudaFuncSetAttribute(k_kv_project, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    k_kv_project<<<2 * p.n_pairs, PTHREADS, bytes, s>>>(p, tx, twk, twv);
    return cudaGetLastError();
}

}  // namespace nvkv
