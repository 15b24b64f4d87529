// Q side of the block-scaled FP4 Q K^T reading (sm_100a): every query row
// quantized to NVFP4 once per visible key frame.
//
// The KV cache is held "in the same format" as the W4A4 generator
// (evermx.com, heading "NVFP4 Quantization End-to-End"), so the logits can
// be taken on FP4 operands.  With K cached after its spatial RoPE
// (nvfp4_kv_append_spatial_rope), RoPE stays relative ("NVlabs LongLive",
// refft.com, Core Analysis block on KV-cache relative RoPE) when the query
// row carries the rest: for a key frame at index f_k, Q_fk is the row with
// its frame segment rotated by f_q - f_k and its spatial segments at its own
// (h, w).  Q_fk is quantized with the cache's block rule under one global
// scale per row, s_gq = fl32(p / 2688), p the row's largest pair magnitude
// fl32(sqrt(fl32(fl32(x^2) + fl32(y^2)))), which no rotation changes.
// The rotations feed the quantizer, so they are fixed in float: cos and sin
// from the host (fp64 angle, rounded once), unfused products and sums; a
// segment at position 0 is left as is.
//
// One thread per (stream, row, head): it loads the row once, finds s_gq and
// writes 72 bytes per visible frame.  This is the quantizer of the reading,
// kept simple; a fused FP4 contraction would form the few frame-dependent
// blocks (channels 0..47) per key tile instead.
#include <cuda_bf16.h>

#include "nvfp4_quant.cuh"
#include "nvkv_internal.h"
#include "ptx.cuh"

namespace nvkv {
namespace {

using namespace q4;

__device__ __forceinline__ void rot(float *x, float2 cs)
{
    const float x0 = x[0], y0 = x[1];
    x[0] = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(y0, cs.y));
    x[1] = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(y0, cs.x));
}

__global__ void __launch_bounds__(128) k_fp4qk_quantize_q(const __grid_constant__ QfkLaunch a)
{
    const int b = blockIdx.y;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)a.Lq * a.H) return;
    const int l = (int)(idx / a.H), h = (int)(idx - (long long)l * a.H);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.q) + (((size_t)b * a.Lq + l) * a.H + h) * 16;
    float q[128];
#pragma unroll
    for (int c = 0; c < 16; ++c) unpack_bf16x8(src[c], q + 8 * c);
    float p = 0.0f;
#pragma unroll
    for (int i = 0; i < 64; ++i)
        p = fmaxf(p, __fsqrt_rn(__fadd_rn(__fmul_rn(q[2 * i], q[2 * i]),
                                          __fmul_rn(q[2 * i + 1], q[2 * i + 1]))));
    float sg = __fdiv_rn(p, 2688.0f);
    if (!(sg >= 1.17549435e-38f)) sg = 1.0f;
    const size_t row = ((size_t)b * a.H + h) * a.Lq + l;
    a.s_gq[row] = sg;
    // spatial segments at the row's own (h, w), the same for every frame
    const int tok = l % a.T, hp = tok / a.grid_w, wp = tok - hp * a.grid_w;
    if (hp != 0)
        for (int i = 0; i < 21; ++i) rot(q + 44 + 2 * i, a.sp[hp * 21 + i]);
    if (wp != 0)
        for (int i = 0; i < 21; ++i) rot(q + 86 + 2 * i, a.sp[(a.grid_h + wp) * 21 + i]);
    const int fq = a.q_pos0[b] + l / a.T;
    for (int j = 0; j < a.n_vis[b]; ++j) {
        float x[48];                             // the frame-dependent blocks 0..2
#pragma unroll
        for (int c = 0; c < 48; ++c) x[c] = q[c];
        const int dpos = fq - a.vis_pos[b][j];
        if (dpos != 0)
            for (int i = 0; i < 22; ++i) rot(x + 2 * i, a.fr[(dpos + kQfkMaxChunk - 1) * 22 + i]);
        uint8_t *codes = a.codes + (row * a.max_vis + j) * 64;
        uint8_t *scales = a.scales + (row * a.max_vis + j) * 8;
#pragma unroll
        for (int blk = 0; blk < 8; ++blk) {
            uint2 c;
            const uint32_t sb = quantize_block_f32(blk < 3 ? x + 16 * blk : q + 16 * blk, sg, c);
            *reinterpret_cast<uint2 *>(codes + blk * 8) = c;
            scales[blk] = (uint8_t)sb;
        }
    }
}

// ------------------------------------------------ the FP4 contraction

// Shared-memory operand layout, K-major without swizzle: 8-row x 16-byte core
// matrices, the four along K of an 8-row group 128 bytes apart (LBO) and the
// 8-row groups 512 bytes apart (SBO); one MMA (K = 64 FP4 = 32 bytes) reads
// two core matrices along K.
constexpr uint32_t kOpBytes = 128 * 64;
__device__ __forceinline__ uint32_t op_off(int r, int chunk)
{
    return (uint32_t)((r >> 3) * 512 + chunk * 128 + (r & 7) * 16);
}

__device__ __forceinline__ uint64_t desc_noswz(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(128u >> 4) << 16;         // LBO: next core matrix along K
    d |= (uint64_t)(512u >> 4) << 32;         // SBO: next 8-row group
    d |= (uint64_t)1 << 46;                   // descriptor version for tcgen05
    return d;                                 // layout type 0: no swizzle
}

// kind::mxf4nvf4, E2M1 x E2M1 -> f32, UE4M3 scales, M = 128, N = 128, both
// K-major, dense, K = 64 per instruction
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_fp4(uint32_t d, uint64_t a, uint64_t b, uint32_t sfa,
                                        uint32_t sfb, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(kIdescFp4), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

// Scale factors of one K step (four 16-element blocks) for 128 rows, in the
// layout the block-scaled MMA reads: column j holds rows 32j .. 32j+31, the
// four block scales of a row in the bytes of its 32-bit word (block order),
// copied into all four 32-lane quarters.  Warp w writes quarter w.
__device__ __forceinline__ void put_scales(uint32_t tcol, const uint32_t *words, int warp)
{
#pragma unroll
    for (int j = 0; j < 4; ++j)
        tmem_st_x1(tcol + ((uint32_t)(warp * 32) << 16) + j, words[j]);
}

// One CTA: 128 query rows x 128 keys of one (b, h).  Per visible frame the
// tile touches, Q_fk of the 128 rows against the tile's 128 K' rows, two
// block-scaled MMAs (K = 128), then the logits of that frame's keys:
// acc * s_gq(row) * s_g(K), in f32.
__global__ void __launch_bounds__(128) k_fp4qk_scores(const __grid_constant__ ScoreLaunch a)
{
    __shared__ __align__(128) uint8_t sA[kOpBytes];
    __shared__ __align__(128) uint8_t sB[kOpBytes];
    __shared__ uint64_t bar;
    __shared__ uint32_t tbase;
    const int t = threadIdx.x, warp = t >> 5;
    const int bh = blockIdx.z, b = bh / a.H, h = bh - b * a.H;
    const int row0 = blockIdx.y * 128, key0 = blockIdx.x * 128;
    const int n_keys = a.n_vis[b] * a.Tr;
    if (key0 >= n_keys) return;                               // uniform per CTA
    if (warp == 0) {
        ptx::tmem_alloc(&tbase, 256);
        ptx::tmem_relinquish();
    }
    if (t == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
    }
    // B: this tile's K' rows (zeros past the visible keys and on padding rows)
    const int key = key0 + t;
    const int kf = key < n_keys ? key / a.Tr : 0, ktok = key - kf * a.Tr;
    const bool kvalid = key < n_keys && ktok < a.Tk;
    const size_t krow = ((size_t)(b * a.H + h)) * a.R + (size_t)a.vis_slot[b][kf] * a.Tr + ktok;
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.k_codes + krow * 64);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w = kvalid ? src[c] : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sB + op_off(t, c)) = w;
        }
    }
    const uint2 ksc = kvalid ? *reinterpret_cast<const uint2 *>(a.k_scales + krow * 8)
                             : make_uint2(0, 0);
    const int row = row0 + t;
    const bool rvalid = row < a.Lq;
    const size_t qrow = ((size_t)(b * a.H + h)) * a.Lq + (rvalid ? row : 0);
    const float sgq = rvalid ? a.s_gq[qrow] : 0.0f;
    const float sgk = a.s_gk[b * a.H + h];
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tbase;
    const uint32_t tD = tmem, tSFA = tmem + 128, tSFB = tmem + 136;
    // B's scales: row = key t of the tile; gather the 32-bit words of rows
    // 32j + lane for this warp's quarter (every quarter holds all rows)
    __shared__ uint2 s_ksc[128], s_qsc[128];
    s_ksc[t] = ksc;
    __syncthreads();
    {
        uint32_t w0[4], w1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w0[j] = s_ksc[32 * j + (t & 31)].x;
            w1[j] = s_ksc[32 * j + (t & 31)].y;
        }
        put_scales(tSFB, w0, warp);
        put_scales(tSFB + 4, w1, warp);
    }
    const int f_first = key0 / a.Tr, f_last = min(n_keys - 1, key0 + 127) / a.Tr;
    uint32_t phase = 0;
    for (int f = f_first; f <= f_last; ++f) {
        // A: Q_f of the 128 rows (zeros past the chunk), and its scales
        const uint8_t *qc = a.q_codes + (qrow * a.max_vis + f) * 64;
        const uint4 *src = reinterpret_cast<const uint4 *>(qc);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w = rvalid ? src[c] : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sA + op_off(t, c)) = w;
        }
        s_qsc[t] = rvalid ? *reinterpret_cast<const uint2 *>(a.q_scales + (qrow * a.max_vis + f) * 8)
                          : make_uint2(0, 0);
        __syncthreads();
        {
            uint32_t w0[4], w1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w0[j] = s_qsc[32 * j + (t & 31)].x;
                w1[j] = s_qsc[32 * j + (t & 31)].y;
            }
            put_scales(tSFA, w0, warp);
            put_scales(tSFA + 4, w1, warp);
        }
        ptx::tmem_wait_st();
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        if (t == 0) {
            const uint32_t a0 = ptx::smem_u32(sA), b0 = ptx::smem_u32(sB);
#pragma unroll
            for (int s = 0; s < 2; ++s)
                mma_fp4(tD, desc_noswz(a0 + 256 * s), desc_noswz(b0 + 256 * s), tSFA + 4 * s,
                        tSFB + 4 * s, s > 0);
            ptx::mma_commit(&bar);
        }
        const int never = 0;
        const bool ok = ptx::mbar_wait(&bar, phase, &never, 2000000000ull);
        if (!__syncthreads_and(ok)) {
            // give the MMAs one more bounded wait before TMEM is released
            if (t == 0) {
                atomicCAS(a.status, 0, (int)NVKV_ERR_TIMEOUT);
                ptx::mbar_wait(&bar, phase, &never, 2000000000ull);
            }
            break;
        }
        phase ^= 1;
        ptx::tc_fence_after();
        // lane t of the accumulator is query row row0 + t; column c key key0 + c
        const uint32_t tq = tD + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            uint32_t v[32];
            ptx::tmem_ld32(tq + q * 32, v);
            ptx::tmem_wait_ld();
            if (rvalid) {
                for (int i = 0; i < 32; ++i) {
                    const int k = key0 + q * 32 + i;
                    if (k >= n_keys || k / a.Tr != f) continue;
                    const int tok = k - f * a.Tr;
                    if (tok >= a.Tk) continue;
                    a.out[(qrow * a.max_vis + f) * a.Tk + tok] =
                        __fmul_rn(__fmul_rn(__uint_as_float(v[i]), sgq), sgk);
                }
            }
        }
        ptx::tc_fence_before();
        __syncthreads();                      // D and the operands are reused by the next frame
        ptx::tc_fence_after();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tbase, 256);
    }
}

}  // namespace

cudaError_t launch_fp4qk_scores(const ScoreLaunch &a, cudaStream_t s)
{
    int max_keys = 0;
    for (int b = 0; b < a.B; ++b) max_keys = max(max_keys, a.n_vis[b] * a.Tr);
    const dim3 grid((unsigned)((max_keys + 127) / 128), (unsigned)((a.Lq + 127) / 128), a.B * a.H);
    k_fp4qk_scores<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_fp4qk_quantize_q(const QfkLaunch &a, cudaStream_t s)
{
    const long long n = (long long)a.Lq * a.H;
    const dim3 grid((unsigned)((n + 127) / 128), a.B);
    k_fp4qk_quantize_q<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace nvkv
