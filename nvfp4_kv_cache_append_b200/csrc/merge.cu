// LSE-weighted merge of partial chunk attentions, sm_100a.
//
// A sequence-parallel KV split ("NVlabs/LongLive 2.0: NVFP4 parallel
// infrastructure for long video generation", section "NVFP4, sequence
// parallel and the async decode path") leaves, per query row, one result per
// shard: O_j = softmax over shard j's keys of the logits, times V, and its
// log normaliser L_j.  The attention over all keys is
//   L = log sum_j exp(L_j),   O = sum_j exp(L_j - L) O_j,
// since the shards' key sets are disjoint.  The parts may live in other GPUs'
// memory mapped into this process: the loads below then cross NVLink, and
// this one kernel is the exchange and the merge.
//
// Layout: 16 threads per (b, q, h) row, each owning 8 channels (one 16-byte
// chunk of every part's bf16 row), so a warp reads two whole 256-byte rows of
// each part.  HBM-bound: n * (256 + 4) bytes read and 256 (+ 4) written per
// row.
//
// The synced form puts the step's cross-rank barrier in the same kernel: each
// CTA first signals every rank that this rank's part is complete (a store
// with release semantics at system scope into that rank's flag array; the
// part was written by earlier work on this stream), then waits for the
// signals of all ranks (acquire loads, bounded in time) before it reads
// their parts.  Any CTA that runs signals, so the barrier cannot deadlock
// on CTAs not yet resident; repeated signals store the same value.  A wait
// that runs out records NVKV_ERR_TIMEOUT in the status word and the CTA
// returns without reading (no trap, the context stays usable).
#include <cuda_bf16.h>

#include "nvkv_internal.h"

namespace nvkv {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_part(const void *base, size_t idx)
{
    // read once, not kept in L1: each chunk of each part is used by one thread
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(static_cast<const uint4 *>(base) + idx));
    return r;
}

__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v)
{
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// signal every rank, then wait for every rank's signal of this epoch; false
// (block-uniform) if a wait ran out or another CTA already reported an error
__device__ bool cross_rank_barrier(const MergeLaunch &m)
{
    const int j = threadIdx.x;
    if (j < m.n) st_release_sys(m.flags[j] + m.rank, m.epoch);
    bool ok = true;
    if (j < m.n && j != m.rank) {
        const uint32_t *f = m.flags[m.rank] + j;
        const volatile int32_t *st = m.status;
        const uint64_t t0 = now_ns();
        // wrap-safe: the flag has reached epoch once (flag - epoch) is
        // non-negative as a signed difference
        while ((int32_t)(ld_acquire_sys(f) - m.epoch) < 0) {
            if (*st != 0) {
                ok = false;
                break;
            }
            if (now_ns() - t0 > m.timeout_ns) {
                atomicCAS(m.status, 0, (int32_t)NVKV_ERR_TIMEOUT);
                ok = false;
                break;
            }
            __nanosleep(256);
        }
    }
    return __syncthreads_and(ok) != 0;
}

__global__ void __launch_bounds__(kThreads) k_lse_merge(const __grid_constant__ MergeLaunch m)
{
    if (m.sync && !cross_rank_barrier(m)) return;
    const long long rows = (long long)m.B * m.nq * m.H;
    const long long r = (long long)blockIdx.x * (kThreads / 16) + (threadIdx.x >> 4);
    if (r >= rows) return;
    const int c = threadIdx.x & 15;                      // 16-byte chunk of the row
    const int h = (int)(r % m.H);
    const long long bq = r / m.H;
    const int q = (int)(bq % m.nq), b = (int)(bq / m.nq);
    const int lq = m.q0 + q;                             // query index in the parts

    float lse[NVKV_MAX_SHARDS];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NVKV_MAX_SHARDS; ++j) {
        if (j < m.n) {
            lse[j] = __ldg(m.lse[j] + ((size_t)b * m.H + h) * m.Lq + lq);
            mx = fmaxf(mx, lse[j]);
        }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float wsum = 0.0f;
    const size_t chunk = (((size_t)b * m.Lq + lq) * m.H + h) * 16 + c;
    if (mx > -INFINITY) {
#pragma unroll
        for (int j = 0; j < NVKV_MAX_SHARDS; ++j) {
            if (j < m.n) {
                const float w = __expf(lse[j] - mx);     // 0 for a part without keys
                if (w > 0.0f) {
                    const uint4 u = ld_part(m.o[j], chunk);
                    const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        acc[2 * i] = fmaf(w, __uint_as_float(p[i] << 16), acc[2 * i]);
                        acc[2 * i + 1] = fmaf(w, __uint_as_float(p[i] & 0xFFFF0000u), acc[2 * i + 1]);
                    }
                    wsum += w;
                }
            }
        }
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        o[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
    reinterpret_cast<uint4 *>(m.out)[(((size_t)b * m.nq + q) * m.H + h) * 16 + c] =
        make_uint4(o[0], o[1], o[2], o[3]);
    if (m.lse_out && c == 0)
        m.lse_out[((size_t)b * m.H + h) * m.nq + q] = wsum > 0.0f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_lse_merge(const MergeLaunch &m, cudaStream_t s)
{
    const long long rows = (long long)m.B * m.nq * m.H;
    const long long blocks = (rows + kThreads / 16 - 1) / (kThreads / 16);
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
    k_lse_merge<<<(unsigned)blocks, kThreads, 0, s>>>(m);
    return cudaGetLastError();
}

}  // namespace nvkv
