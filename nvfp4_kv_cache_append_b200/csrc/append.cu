// NVFP4 quantize-append and bf16 append kernels (sm_100a).
//
// In-place quantized KV-cache update ("NVlabs/LongLive 2.0: NVFP4 parallel
// infrastructure for long video generation", section "NVFP4, sequence
// parallel and the async decode path").  Format: E2M1 codes, one E4M3 scale
// per 16 head_dim elements, one FP32 global scale per (K/V, batch, head):
//   s_g  = fl32(amax(first chunk) / 2688)        (1 if not a normal float)
//   s_b  = E4M3_RNE(min(fl32(amax16 / fl32(6 s_g)), 448))
//   q_i  = E2M1_RNE_sat(fl32(x_i / fl32(s_b s_g)))   (s_b = 0 -> all zero)
// Element 2i is the low nibble of byte i; a magnitude that rounds to zero is
// stored as code 0.  The FP32 operations are IEEE round-to-nearest (no
// contraction, true division), so the codes are bit-exact.
//
// Memory: HBM-bound.  Each thread owns two adjacent 16-element blocks: four
// 16-byte loads of bf16 input (a warp reads 2 KB contiguous), one 16-byte
// code store and one 2-byte scale store (four threads of a token-head write
// its 64 contiguous code bytes).  Rows go straight into the physical frame
// slot (no staging).
//
// The 16 quotients x_i / (s_b s_g) of a block share their divisor, so they
// are taken by Markstein's correctly rounded division (P. Markstein, "IA-64
// and Elementary Functions", 2000: with r = RN(1/d) and q = RN(x r), the
// residual e = x - q d is exact under an FMA and RN(q + e r) = RN(x / d)):
// one reciprocal per block, three FMA-pipe operations per element.  The
// theorem needs the residual representable, which holds for 2^-64 <= d <=
// 2^64 and quotients below 2^64 whenever |x / d| >= 1/16; below 1/16 every
// candidate quotient encodes to code 0.  Blocks outside that range (tiny or
// huge scales, infinities, NaN) take IEEE division.
#include <cuda_bf16.h>

#include "nvfp4_quant.cuh"
#include "nvkv_internal.h"

namespace nvkv {
namespace {

using namespace q4;


__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// l / Ts for 0 <= l < 2^24 by a float reciprocal with a one-step fix-up
__device__ __forceinline__ int frame_of(int l, const AppendLaunch &a)
{
    int f = __float2int_rz((float)l * a.inv_Ts);
    if (f * a.Ts > l) --f;
    else if ((f + 1) * a.Ts <= l) ++f;
    return f;
}

// amax of the first chunk per (K/V, batch, head).  blockDim = (8H, ty),
// grid = (gx, 2B).  amax must be zero on entry; float bits of non-negative
// values order like unsigned integers, so atomicMax on the bits is exact.
__global__ void k_first_chunk_amax(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                   uint32_t *__restrict__ amax, int B, int H, int Lq)
{
    __shared__ uint32_t s_max[64];
    const int tid = threadIdx.y * blockDim.x + threadIdx.x;
    if (tid < H) s_max[tid] = 0u;
    __syncthreads();
    const int t = blockIdx.y / B, b = blockIdx.y - t * B;
    const uint4 *src = t ? v : k;
    const int h = threadIdx.x >> 3, blk = threadIdx.x & 7;
    uint32_t m = 0u;
    for (int l = blockIdx.x * blockDim.y + threadIdx.y; l < Lq; l += gridDim.x * blockDim.y) {
        const uint4 *p = src + (((size_t)b * Lq + l) * H + h) * 16 + blk * 2;
        m = __vmaxu2(m, __vmaxu2(absmax_bits(ld_stream(p)), absmax_bits(ld_stream(p + 1))));
    }
    uint32_t f = __float_as_uint(halves_max(m));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
        const uint32_t g = __shfl_xor_sync(0xFFFFFFFFu, f, o);
        f = g > f ? g : f;
    }
    if (blk == 0) atomicMax(&s_max[h], f);
    __syncthreads();
    if (tid < H && s_max[tid]) atomicMax(&amax[(t * B + b) * H + tid], s_max[tid]);
}

// Quantize the two blocks (elements 32 pair .. 32 pair + 31) of one
// token-head row given as four 16-byte words, and write codes and scales
// into cache row `row`.
__device__ __forceinline__ void quantize_pair(const AppendLaunch &a, int t, int h, int pr,
                                              size_t row, float sg, uint4 w0, uint4 w1, uint4 w2,
                                              uint4 w3)
{
    uint2 c0, c1;
    const uint32_t s0 = quantize_block(w0, w1, sg, c0);
    const uint32_t s1 = quantize_block(w2, w3, sg, c1);
    *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(t ? a.v_data : a.k_data) + row * 64 + pr * 16) =
        make_uint4(c0.x, c0.y, c1.x, c1.y);
    *reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(t ? a.v_scales : a.k_scales) + row * 8 +
                                  pr * 2) = (uint16_t)(s0 | (s1 << 8));
}

__device__ __forceinline__ float head_scale(const AppendLaunch &a, int gi, bool writer)
{
    if (a.first) {
        const float sg = global_scale_from_amax(a.amax[gi]);
        if (writer) a.s_g[gi] = sg;
        return sg;
    }
    return a.s_g[gi];
}

// blockDim = (4H, ty): threadIdx.x = h * 4 + pair (blocks 2 pair, 2 pair + 1
// of the token-head: 64 bytes in, 16 code bytes and 2 scale bytes out),
// threadIdx.y = token in the CTA's token group.  grid = (ceil(C Ts / ty), 2B):
// blockIdx.y = t * B + b with t = 0 for K and 1 for V.  Row l of the grid is
// token tok_off + l % Ts of chunk frame l / Ts (all tokens: Ts = T), stored
// in row l % Ts of its frame's slot (Tr rows per slot; the padding row of an
// odd Ts is never written).
__global__ void __launch_bounds__(512) k_nvfp4_append(const __grid_constant__ AppendLaunch a)
{
    const int t = blockIdx.y / a.B, b = blockIdx.y - t * a.B;
    const int l = blockIdx.x * blockDim.y + threadIdx.y;
    if (l >= a.C * a.Ts) return;
    const int h = threadIdx.x >> 2, pr = threadIdx.x & 3;
    const int frame = frame_of(l, a), tok = l - frame * a.Ts;
    const int src_l = frame * a.T + a.tok_off + tok;
    const uint4 *src = reinterpret_cast<const uint4 *>(t ? a.v : a.k) +
                       (((size_t)b * a.Lq + src_l) * a.H + h) * 16 + pr * 4;
    const uint4 w0 = ld_stream(src), w1 = ld_stream(src + 1);
    const uint4 w2 = ld_stream(src + 2), w3 = ld_stream(src + 3);
    const int gi = (t * a.B + b) * a.H + h;
    const float sg = head_scale(a, gi, l == 0 && pr == 0);
    const int slot = a.slot[b * a.C + frame];
    quantize_pair(a, t, h, pr, (size_t)(b * a.H + h) * a.R + (size_t)slot * a.Tr + tok, sg, w0, w1,
                  w2, w3);
}

// bf16 twin: blockDim = (16H, ty), one 16-byte chunk per thread; rows as in
// k_nvfp4_append.
__global__ void __launch_bounds__(1024) k_bf16_append(const __grid_constant__ AppendLaunch a)
{
    const int t = blockIdx.y / a.B, b = blockIdx.y - t * a.B;
    const int l = blockIdx.x * blockDim.y + threadIdx.y;
    if (l >= a.C * a.Ts) return;
    const int h = threadIdx.x >> 4, c = threadIdx.x & 15;
    const int frame = frame_of(l, a), tok = l - frame * a.Ts;
    const uint4 *src = reinterpret_cast<const uint4 *>(t ? a.v : a.k) +
                       (((size_t)b * a.Lq + frame * a.T + a.tok_off + tok) * a.H + h) * 16 + c;
    const int slot = a.slot[b * a.C + frame];
    const size_t row = (size_t)(b * a.H + h) * a.R + (size_t)slot * a.Tr + tok;
    reinterpret_cast<uint4 *>(t ? a.v_data : a.k_data)[row * 16 + c] = ld_stream(src);
}

// ------------------------------------------- K with its spatial RoPE applied

// Rotate the pairs of n consecutive channels starting at channel ch0 (even)
// that lie in the h segment [44, 86) or the w segment [86, 128), in float:
// (fl(fl(x c) - fl(y s)), fl(fl(x s) + fl(y c))), no contraction; the frame
// segment [0, 44) is left as is.
__device__ __forceinline__ void rotate_spatial(float *x, int n, int ch0, int hp, int wp,
                                               const SpatialRope &R)
{
    for (int j = 0; j < n; j += 2) {
        const int ch = ch0 + j;
        if (ch < 44) continue;
        const float2 cs = ch < 86 ? R.h[hp * 21 + ((ch - 44) >> 1)] : R.w[wp * 21 + ((ch - 86) >> 1)];
        const float x0 = x[j], y0 = x[j + 1];
        x[j] = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(y0, cs.y));
        x[j + 1] = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(y0, cs.x));
    }
}

// k_first_chunk_amax with K's spatial pairs rotated first (row l of the chunk
// is token l % T of its frame, at (h, w) = divmod(l % T, grid_w))
__global__ void k_first_chunk_amax_rope(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                        uint32_t *__restrict__ amax, int B, int H, int Lq, int T,
                                        int grid_w, const __grid_constant__ SpatialRope R)
{
    __shared__ uint32_t s_max[64];
    const int tid = threadIdx.y * blockDim.x + threadIdx.x;
    if (tid < H) s_max[tid] = 0u;
    __syncthreads();
    const int t = blockIdx.y / B, b = blockIdx.y - t * B;
    const uint4 *src = t ? v : k;
    const int h = threadIdx.x >> 3, blk = threadIdx.x & 7;
    float m = 0.0f;
    for (int l = blockIdx.x * blockDim.y + threadIdx.y; l < Lq; l += gridDim.x * blockDim.y) {
        const uint4 *p = src + (((size_t)b * Lq + l) * H + h) * 16 + blk * 2;
        float x[16];
        unpack_bf16x8(ld_stream(p), x);
        unpack_bf16x8(ld_stream(p + 1), x + 8);
        if (t == 0) {
            const int tok = l % T;
            rotate_spatial(x, 16, blk * 16, tok / grid_w, tok % grid_w, R);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(x[i]));
    }
    uint32_t f = __float_as_uint(m);
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
        const uint32_t g = __shfl_xor_sync(0xFFFFFFFFu, f, o);
        f = g > f ? g : f;
    }
    if (blk == 0) atomicMax(&s_max[h], f);
    __syncthreads();
    if (tid < H && s_max[tid]) atomicMax(&amax[(t * B + b) * H + tid], s_max[tid]);
}

// k_nvfp4_append with K's spatial pairs rotated in float before quantizing
// (the cache layout of the block-scaled FP4 Q K^T contraction); V as is.
__global__ void __launch_bounds__(512) k_nvfp4_append_rope(const __grid_constant__ AppendLaunch a,
                                                           const __grid_constant__ SpatialRope R)
{
    const int t = blockIdx.y / a.B, b = blockIdx.y - t * a.B;
    const int l = blockIdx.x * blockDim.y + threadIdx.y;
    if (l >= a.C * a.Ts) return;
    const int h = threadIdx.x >> 2, pr = threadIdx.x & 3;
    const int frame = frame_of(l, a), tok = l - frame * a.Ts;
    const int src_l = frame * a.T + a.tok_off + tok;
    const uint4 *src = reinterpret_cast<const uint4 *>(t ? a.v : a.k) +
                       (((size_t)b * a.Lq + src_l) * a.H + h) * 16 + pr * 4;
    const uint4 w0 = ld_stream(src), w1 = ld_stream(src + 1);
    const uint4 w2 = ld_stream(src + 2), w3 = ld_stream(src + 3);
    const int gi = (t * a.B + b) * a.H + h;
    const float sg = head_scale(a, gi, l == 0 && pr == 0);
    const int slot = a.slot[b * a.C + frame];
    const size_t row = (size_t)(b * a.H + h) * a.R + (size_t)slot * a.Tr + tok;
    if (t == 1) {
        quantize_pair(a, t, h, pr, row, sg, w0, w1, w2, w3);
        return;
    }
    float x[32];
    unpack_bf16x8(w0, x);
    unpack_bf16x8(w1, x + 8);
    unpack_bf16x8(w2, x + 16);
    unpack_bf16x8(w3, x + 24);
    const int ft = a.tok_off + tok;
    rotate_spatial(x, 32, pr * 32, ft / a.grid_w, ft % a.grid_w, R);
    uint2 c0, c1;
    const uint32_t s0 = quantize_block_f32(x, sg, c0);
    const uint32_t s1 = quantize_block_f32(x + 16, sg, c1);
    *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.k_data) + row * 64 + pr * 16) =
        make_uint4(c0.x, c0.y, c1.x, c1.y);
    *reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(a.k_scales) + row * 8 + pr * 2) =
        (uint16_t)(s0 | (s1 << 8));
}

__global__ void k_encode_e2m1(const float *__restrict__ y, uint8_t *__restrict__ out, size_t n)
{
    const size_t i0 = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (i0 >= n) return;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (i0 + j < n) ? y[i0 + j] : 0.0f;
    const uint32_t w = drop_negative_zero(e2m1x8(v));
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (i0 + j < n) out[i0 + j] = (w >> (4 * j)) & 15u;
}

__global__ void k_encode_block_scale(const float *__restrict__ t, uint8_t *__restrict__ out,
                                     size_t n)
{
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = (uint8_t)e4m3_code(t[i]);
}

dim3 append_block(int H, int per_head)
{
    const int x = per_head * H;
    const int y = x >= 256 ? 1 : 256 / x;
    return dim3(x, y);
}

}  // namespace

cudaError_t launch_nvfp4_append(const AppendLaunch &a_in, cudaStream_t s)
{
    AppendLaunch a = a_in;
    a.inv_Ts = 1.0f / (float)a.Ts;
    const dim3 blk = append_block(a.H, 4);
    if (a.first) {
        cudaError_t e = cudaMemsetAsync(a.amax, 0, sizeof(uint32_t) * 2 * a.B * a.H, s);
        if (e != cudaSuccess) return e;
        const dim3 blk8 = append_block(a.H, 8);
        const unsigned gx = (a.Lq + blk8.y - 1) / blk8.y;
        const dim3 g2(gx < 148 ? gx : 148, 2 * a.B);
        k_first_chunk_amax<<<g2, blk8, 0, s>>>(static_cast<const uint4 *>(a.k),
                                              static_cast<const uint4 *>(a.v), a.amax, a.B, a.H,
                                              a.Lq);
    }
    const dim3 grid((a.C * a.Ts + blk.y - 1) / blk.y, 2 * a.B);
    k_nvfp4_append<<<grid, blk, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_append_rope(const AppendLaunch &a_in, const SpatialRope &r, cudaStream_t s)
{
    AppendLaunch a = a_in;
    a.inv_Ts = 1.0f / (float)a.Ts;
    const dim3 blk = append_block(a.H, 4);
    if (a.first) {
        cudaError_t e = cudaMemsetAsync(a.amax, 0, sizeof(uint32_t) * 2 * a.B * a.H, s);
        if (e != cudaSuccess) return e;
        const dim3 blk8 = append_block(a.H, 8);
        const unsigned gx = (a.Lq + blk8.y - 1) / blk8.y;
        const dim3 g2(gx < 148 ? gx : 148, 2 * a.B);
        k_first_chunk_amax_rope<<<g2, blk8, 0, s>>>(static_cast<const uint4 *>(a.k),
                                                   static_cast<const uint4 *>(a.v), a.amax, a.B,
                                                   a.H, a.Lq, a.T, a.grid_w, r);
    }
    const dim3 grid((a.C * a.Ts + blk.y - 1) / blk.y, 2 * a.B);
    k_nvfp4_append_rope<<<grid, blk, 0, s>>>(a, r);
    return cudaGetLastError();
}

cudaError_t launch_bf16_append(const AppendLaunch &a_in, cudaStream_t s)
{
    AppendLaunch a = a_in;
    a.inv_Ts = 1.0f / (float)a.Ts;
    const dim3 blk = append_block(a.H, 16);
    const dim3 grid((a.C * a.Ts + blk.y - 1) / blk.y, 2 * a.B);
    k_bf16_append<<<grid, blk, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_encode_e2m1(const float *y, uint8_t *codes, size_t n, cudaStream_t s)
{
    const size_t groups = (n + 7) / 8;
    k_encode_e2m1<<<(unsigned)((groups + 255) / 256), 256, 0, s>>>(y, codes, n);
    return cudaGetLastError();
}

cudaError_t launch_encode_block_scale(const float *t, uint8_t *codes, size_t n, cudaStream_t s)
{
    k_encode_block_scale<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(t, codes, n);
    return cudaGetLastError();
}

}  // namespace nvkv
