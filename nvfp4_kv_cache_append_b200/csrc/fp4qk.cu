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

}  // namespace

cudaError_t launch_fp4qk_quantize_q(const QfkLaunch &a, cudaStream_t s)
{
    const long long n = (long long)a.Lq * a.H;
    const dim3 grid((unsigned)((n + 127) / 128), a.B);
    k_fp4qk_quantize_q<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace nvkv
