// LSE merge of two partial attentions over disjoint key sets.
//
// "ISPA" (Absorción Paramétrica Específica de Instancia), §2.1 Dual-Stream Warmup and
// contribution 2: the per-row log-sum-exp kept by attention kernels lets attention be
// split into a local and a history branch and fused afterwards.  Per row, with
// M = max(L1, L2):  L = M + ln(e^{L1-M} + e^{L2-M}),  O = e^{L1-L} O1 + e^{L2-L} O2.
//
// Memory-bound: each row reads 2 x (d bf16 + 1 fp32) and writes d bf16 + 1 fp32.
// A group of d/8 threads owns a row, every thread moves 16 bytes of each O; each thread
// takes RPT rows, all their loads issued before any arithmetic.
#include <cstdint>

#include "sfa.h"
#include "sfa_internal.h"
#include "sfa_ptx.cuh"

namespace sfa {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t to_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(int64_t rows, const uint4 *__restrict__ o1,
                                                        const float *__restrict__ lse1,
                                                        const uint4 *__restrict__ o2,
                                                        const float *__restrict__ lse2, uint4 *o, float *lse)
{
    constexpr int G = D / 8;  // threads per row
    constexpr int RPT = 2;  // rows per thread (measured: 2 beat 1 and 4 on 2M rows)
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int sub = threadIdx.x % G;
    const int64_t row_stride = (int64_t)gridDim.x * blockDim.x / G;
    const unsigned group = ((1u << G) - 1u) << ((threadIdx.x % 32) & ~(G - 1));
    for (int64_t r0 = gtid / G; r0 < rows; r0 += row_stride * RPT) {
        uint4 a[RPT], b[RPT];
        float l1[RPT], l2[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int64_t r = r0 + k * row_stride;
            l1[k] = 0.f;
            l2[k] = 0.f;
            if (r < rows) {
                a[k] = o1[r * G + sub];
                b[k] = o2[r * G + sub];
                if (sub == 0) {
                    l1[k] = lse1[r];
                    l2[k] = lse2[r];
                }
            }
        }
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int64_t r = r0 + k * row_stride;
            if (r >= rows) break;
            const float x1 = __shfl_sync(group, l1[k], 0, G);
            const float x2 = __shfl_sync(group, l2[k], 0, G);
            const float m = fmaxf(x1, x2);
            float w1 = 0.f, w2 = 0.f, L = -INFINITY;
            if (m != -INFINITY) {
                const float e1 = x1 == -INFINITY ? 0.f : expf(x1 - m);
                const float e2 = x2 == -INFINITY ? 0.f : expf(x2 - m);
                const float sm = e1 + e2;
                L = m + logf(sm);
                w1 = e1 / sm;
                w2 = e2 / sm;
            }
            const uint32_t av[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
            const uint32_t bv[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
            uint32_t ov[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = w1 * bf16_lo(av[i]) + w2 * bf16_lo(bv[i]);
                const float hi = w1 * bf16_hi(av[i]) + w2 * bf16_hi(bv[i]);
                ov[i] = to_bf16x2(lo, hi);
            }
            o[r * G + sub] = make_uint4(ov[0], ov[1], ov[2], ov[3]);
            if (sub == 0) lse[r] = L;
        }
    }
}

// k-way merge of split-KV partial results (the same LSE rule applied to S branches):
// o_part bf16 [S][rows][D] and lse_part fp32 [S][rows] (rows = B*H*Lq in (b, h, i)
// order) -> O at o + b*os0 + h*os1 + i*os2 and LSE [rows].  D/8 threads per row, the
// lane s of a row's group holds branch s's weight (S <= D/8).
template <int D>
__global__ void __launch_bounds__(256) lse_combine_kernel(int64_t rows, int S, int S1, int H, int64_t Lq,
                                                          const uint4 *__restrict__ o_part,
                                                          const float *__restrict__ lse_part, uint16_t *o,
                                                          int64_t os0, int64_t os1, int64_t os2, float *lse,
                                                          uint16_t *o1, float *lse1)
{
    pdl_wait();  // launched as a dependent of the forward kernel that writes the partials
    // Merges slices [0, S) of the partials into (o, lse) and, when o1 is set, slices
    // [0, S1) into (o1, lse1) (same strides): one group of D/8 threads per row, lane `sub`
    // of the group holds slice `sub`'s LSE.
    constexpr int G = D / 8;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int sub = threadIdx.x % G;
    const unsigned group = ((1u << G) - 1u) << ((threadIdx.x % 32) & ~(G - 1));
    const int64_t row_stride = (int64_t)gridDim.x * blockDim.x / G;
    for (int64_t r = gtid / G; r < rows; r += row_stride) {
        const float ls = sub < S ? lse_part[(int64_t)sub * rows + r] : -INFINITY;
        const float ls1 = sub < S1 ? ls : -INFINITY;
        float m = ls, m1 = ls1;
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) {
            m = fmaxf(m, __shfl_xor_sync(group, m, off, G));
            m1 = fmaxf(m1, __shfl_xor_sync(group, m1, off, G));
        }
        const float w = (ls == -INFINITY) ? 0.f : expf(ls - m);
        const float w1 = (ls1 == -INFINITY) ? 0.f : expf(ls1 - m1);
        float tot = w, tot1 = w1;
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) {
            tot += __shfl_xor_sync(group, tot, off, G);
            tot1 += __shfl_xor_sync(group, tot1, off, G);
        }
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float acc1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int sidx = 0; sidx < S; ++sidx) {
            const float ws = __shfl_sync(group, w, sidx, G);
            const float ws1 = __shfl_sync(group, w1, sidx, G);
            if (ws != 0.f || ws1 != 0.f) {
                const uint4 v = o_part[((int64_t)sidx * rows + r) * G + sub];
                const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] += ws * bf16_lo(vv[i]);
                    acc[2 * i + 1] += ws * bf16_hi(vv[i]);
                    acc1[2 * i] += ws1 * bf16_lo(vv[i]);
                    acc1[2 * i + 1] += ws1 * bf16_hi(vv[i]);
                }
            }
        }
        const int64_t b = r / ((int64_t)H * Lq), h = (r / Lq) % H, i = r % Lq;
        const int64_t off = b * os0 + h * os1 + i * os2 + sub * 8;
        {
            const bool empty = (m == -INFINITY);
            const float inv = empty ? 0.f : 1.f / tot;
            uint4 out;
            out.x = to_bf16x2(acc[0] * inv, acc[1] * inv);
            out.y = to_bf16x2(acc[2] * inv, acc[3] * inv);
            out.z = to_bf16x2(acc[4] * inv, acc[5] * inv);
            out.w = to_bf16x2(acc[6] * inv, acc[7] * inv);
            *reinterpret_cast<uint4 *>(o + off) = out;
            if (sub == 0) lse[r] = empty ? -INFINITY : m + logf(tot);
        }
        if (o1) {
            const bool empty = (m1 == -INFINITY);
            const float inv = empty ? 0.f : 1.f / tot1;
            uint4 out;
            out.x = to_bf16x2(acc1[0] * inv, acc1[1] * inv);
            out.y = to_bf16x2(acc1[2] * inv, acc1[3] * inv);
            out.z = to_bf16x2(acc1[4] * inv, acc1[5] * inv);
            out.w = to_bf16x2(acc1[6] * inv, acc1[7] * inv);
            *reinterpret_cast<uint4 *>(o1 + off) = out;
            if (sub == 0) lse1[r] = empty ? -INFINITY : m1 + logf(tot1);
        }
    }
}

}  // namespace

sfa_status launch_lse_combine(int64_t rows, int S, int d, int H, int64_t Lq, const void *o_part,
                              const float *lse_part, void *o, const int64_t *o_stride, float *lse, cudaStream_t s,
                              int S1, void *o1, float *lse1)
{
    if (rows == 0) return SFA_OK;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    const int64_t need = (rows * (d / 8) + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;
    const int blocks = (int)(need < cap ? need : cap);
    // a programmatic dependent of the forward kernel before it on the stream: its CTAs take
    // the SMs that kernel leaves and wait there for its partials
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e =
        d == 128 ? cudaLaunchKernelEx(&cfg, lse_combine_kernel<128>, rows, S, S1, H, Lq, (const uint4 *)o_part, lse_part,
                                      (uint16_t *)o, o_stride[0], o_stride[1], o_stride[2], lse, (uint16_t *)o1, lse1)
                 : cudaLaunchKernelEx(&cfg, lse_combine_kernel<64>, rows, S, S1, H, Lq, (const uint4 *)o_part, lse_part,
                                      (uint16_t *)o, o_stride[0], o_stride[1], o_stride[2], lse, (uint16_t *)o1, lse1);
    if (e != cudaSuccess) return SFA_ERR_CUDA;
    return launch_status();
}

}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_lse_merge(int64_t rows, int32_t d, const void *o1, const float *lse1,
                                    const void *o2, const float *lse2, void *o, float *lse,
                                    sfa_stream_t stream)
{
    if (rows < 0) return SFA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SFA_ERR_UNSUPPORTED;
    if (rows == 0) return SFA_OK;
    if (!o1 || !o2 || !o || !lse1 || !lse2 || !lse) return SFA_ERR_INVALID_ARG;
    for (const void *p : {o1, o2, (const void *)o})
        if (reinterpret_cast<uintptr_t>(p) % 16) return SFA_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    const int64_t need = (rows * (d / 8) + threads * 2 - 1) / (threads * 2);  // two rows per thread
    const int64_t cap = (int64_t)sms * 8;  // 8 resident blocks of 256 threads per SM
    const int blocks = (int)(need < cap ? need : cap);
    cudaStream_t s = as_cuda(stream);
    if (d == 128)
        lse_merge_kernel<128><<<blocks, threads, 0, s>>>(rows, (const uint4 *)o1, lse1, (const uint4 *)o2,
                                                         lse2, (uint4 *)o, lse);
    else
        lse_merge_kernel<64><<<blocks, threads, 0, s>>>(rows, (const uint4 *)o1, lse1, (const uint4 *)o2,
                                                        lse2, (uint4 *)o, lse);
    return launch_status();
}
