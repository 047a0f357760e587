// Hierarchical sparse attention (HSA): the two-level selection of key blocks.
//
// "Resumen Técnico: LIGHT FORCING", §2.2 Atención Dispersa Jerárquica: query and key
// tokens are mean-pooled per block and per frame (token compression); each query block
// retrieves a few history frames with the frame-level pooled keys (frame selection), then
// the critical blocks inside those frames with the block-level pooled keys (block
// selection); attention then runs over the selected frame-block pairs only
// (sfa_forward_blocks, in sfa_forward.cu).
//
// Two kernels:
//   * hsa_pool_kernel: one CTA per 128-token key block; 16-byte loads, four rows of them
//     in flight per thread, fp32 sums per column, one mean per block.
//     HBM-bound: every K and Q element is read once.  hsa_frame_mean_kernel then forms
//     each frame's mean as the token-weighted average of its block means.
//   * hsa_select_kernel: one CTA per (b, h, t, query block): the mean of its query rows
//     (the same pooling code), scores of the history
//     frames, top k_frames, scores of their blocks, top k_blocks (a candidate is kept
//     when fewer than k candidates rank before it: one pass, no serial rounds), then the
//     sorted union with the always-attended blocks, compacted with a block-wide prefix
//     count.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "sfa.h"
#include "sfa_internal.h"

namespace sfa {
namespace {

constexpr int KEY_BLOCK = 128;    // tokens per key block
constexpr int QUERY_BLOCK = 256;  // query rows per query block
constexpr int POOL_THREADS = 256;
constexpr int SELECT_THREADS = 256;
constexpr int MAX_ENTRIES = 65536;  // T_kv * nblk bound (the block flags live in shared memory)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Mean of rows [r0, r1) of one frame, per column: `frame` points at the frame's first row
// (row stride s_row elements).  POOL_THREADS threads: D/8 per row (8 columns, one 16-byte
// load each), POOL_THREADS / (D/8) rows per round and UNROLL rounds of loads in flight, then
// the row groups are added in order through `part`; threads < D write out[column].  Each
// thread adds its rows in row order whatever UNROLL is, so every UNROLL gives the same means.
template <int D, int UNROLL>
__device__ __forceinline__ void pool_segment(const uint16_t *frame, int64_t s_row, int r0, int r1,
                                             float (*part)[D], float *out)
{
    constexpr int TPR = D / 8;                 // threads per row
    constexpr int RG = POOL_THREADS / TPR;     // rows per load round
    const int cg = threadIdx.x % TPR, rg = threadIdx.x / TPR;
    const uint16_t *base = frame + cg * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r = r0 + rg; r < r1; r += UNROLL * RG) {
        uint4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
            if (r + u * RG < r1) v[u] = __ldg(reinterpret_cast<const uint4 *>(base + (int64_t)(r + u * RG) * s_row));
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            if (r + u * RG < r1) {
                acc[0] += bf16_lo(v[u].x);
                acc[1] += bf16_hi(v[u].x);
                acc[2] += bf16_lo(v[u].y);
                acc[3] += bf16_hi(v[u].y);
                acc[4] += bf16_lo(v[u].z);
                acc[5] += bf16_hi(v[u].z);
                acc[6] += bf16_lo(v[u].w);
                acc[7] += bf16_hi(v[u].w);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) part[rg][cg * 8 + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < D) {
        float sum = 0.f;
        for (int g = 0; g < RG; ++g) sum += part[g][threadIdx.x];
        out[threadIdx.x] = sum / (float)(r1 - r0);
    }
    __syncthreads();
}

// Pooling launch: segment means of the keys (KEY_BLOCK rows) and/or the queries
// (QUERY_BLOCK rows).  CTA x of grid row bh = b*H + h takes key segment x (x < nk =
// nblk * T_kv when the keys are pooled: segment x % nblk of frame x / nblk) or query
// segment x - nk, and writes its mean to out[((bh * n_frames + f) * nseg + sg)][D] of its
// tensor; the last segment of a frame holds the remaining rows.
struct PoolArgs {
    const uint16_t *k, *q;
    int64_t k_sb, k_sh, k_sr, q_sb, q_sh, q_sr;  // strides in elements
    int H, P, T_kv, Tq, nblk, nqb;
    int k_on;  // 1: the launch pools the keys (the first nblk * T_kv CTAs of a row), 0: queries only
    float *kb, *qb;
};

template <int D>
__global__ void __launch_bounds__(POOL_THREADS) hsa_pool_kernel(const __grid_constant__ PoolArgs a)
{
    __shared__ float part[POOL_THREADS / (D / 8)][D];
    const int bh = blockIdx.y;
    const int nk = a.k_on ? a.nblk * a.T_kv : 0;
    const bool is_k = (int)blockIdx.x < nk;
    const int x = is_k ? blockIdx.x : blockIdx.x - nk;
    const int nseg = is_k ? a.nblk : a.nqb, seg = is_k ? KEY_BLOCK : QUERY_BLOCK;
    const int sg = x % nseg, f = x / nseg;
    const int n_frames = is_k ? a.T_kv : a.Tq;
    const int r0 = sg * seg, r1 = min(r0 + seg, a.P);
    const int64_t s_b = is_k ? a.k_sb : a.q_sb, s_h = is_k ? a.k_sh : a.q_sh, s_row = is_k ? a.k_sr : a.q_sr;
    const uint16_t *frame = (is_k ? a.k : a.q) + (int64_t)(bh / a.H) * s_b + (int64_t)(bh % a.H) * s_h +
                            (int64_t)f * a.P * s_row;
    float *out = (is_k ? a.kb : a.qb) + (((int64_t)bh * n_frames + f) * nseg + sg) * D;
    pool_segment<D, 4>(frame, s_row, r0, r1, part, out);
}

// Frame means from the block means: the token-weighted average of a frame's blocks.
// One thread per (b*H + h, frame, column).
template <int D>
__global__ void hsa_frame_mean_kernel(const float *kb, int64_t n, int P, int nblk, float *kf)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int64_t fr = i / D, c = i % D;
    const float *src = kb + fr * nblk * D + c;
    float s = 0.f;
    for (int b = 0; b < nblk; ++b) s += src[(int64_t)b * D] * (float)(min(b * KEY_BLOCK + KEY_BLOCK, P) - b * KEY_BLOCK);
    kf[i] = s / (float)P;
}

struct SelectArgs {
    int B, H, Tq, T_kv, P, nblk, nqb, Amax;
    int q_off, n_sink, n_prev, chunk_len, k_frames, k_blocks;
    const float *kf;  // [B][H][T_kv][D]
    const float *kb;  // [B][H][T_kv][nblk][D]
    const uint16_t *q;         // bf16 queries: the CTA pools its own query block
    int64_t q_sb, q_sh, q_sr;  // strides in elements
    int32_t *blocks;  // [B][H][Tq][nqb][Amax]
    int32_t *counts;  // [B][H][Tq][nqb]
};

// a > b in the selection order: larger score, then smaller id
__device__ __forceinline__ bool ranks_before(float sa, int ia, float sb, int ib)
{
    return sa > sb || (sa == sb && ia < ib);
}

// Number of the n candidates that rank before candidate (s, id): its position in the
// selection order (top-k keeps the candidates whose position is below k).
__device__ __forceinline__ int rank_of(const float *scores, const int *ids, int n, float s, int id)
{
    int r = 0;
    for (int j = 0; j < n; ++j) r += ranks_before(scores[j], ids[j], s, id) ? 1 : 0;
    return r;
}

// dot(q, key_b) of D floats for NB keys by one warp: the loads of all NB keys are issued
// before any sum, so the warp waits for L2 once per NB dots.  Each lane adds its D / 32
// products in order, then a butterfly adds the lanes: equal inputs give equal scores.
template <int D, int NB>
__device__ __forceinline__ void warp_dots(const float *q, const float *const (&key)[NB], const bool (&on)[NB],
                                          float (&res)[NB])
{
    const int lane = threadIdx.x & 31;
    float kv[NB][D / 32];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) kv[b][i] = on[b] ? __ldg(key[b] + lane + 32 * i) : 0.f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) s = fmaf(q[lane + 32 * i], kv[b][i], s);
        res[b] = s;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int b = 0; b < NB; ++b) res[b] += __shfl_xor_sync(0xffffffffu, res[b], off);
}

// Dynamic shared memory: frame scores/ids [T_kv], block scores/ids [k_frames' * nblk],
// selected frames, frame flags [T_kv], entry flags [T_kv * nblk].
template <int D>
__global__ void __launch_bounds__(SELECT_THREADS, 2) hsa_select_kernel(const __grid_constant__ SelectArgs a)
{
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ float qv[D];
    __shared__ int n_hist_s, n_sel_s;
    __shared__ int warp_tot[SELECT_THREADS / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = SELECT_THREADS / 32;
    int u = blockIdx.x;
    const int qi = u % a.nqb;
    u /= a.nqb;
    const int t = u % a.Tq;
    u /= a.Tq;
    const int h = u % a.H;
    const int b = u / a.H;
    const int n_sel_max = min(a.k_frames, a.T_kv);
    const int n_bc_max = n_sel_max * a.nblk;
    const int n_entries = a.T_kv * a.nblk;
    float *f_score = reinterpret_cast<float *>(sm);
    int *f_id = reinterpret_cast<int *>(f_score + a.T_kv);
    float *b_score = reinterpret_cast<float *>(f_id + a.T_kv);
    int *b_id = reinterpret_cast<int *>(b_score + n_bc_max);
    int *sel = b_id + n_bc_max;                                         // [n_sel_max]
    uint8_t *f_taken = reinterpret_cast<uint8_t *>(sel + n_sel_max);   // [T_kv]
    uint8_t *flag = f_taken + a.T_kv;                                   // [n_entries]

    const int c = t + a.q_off;
    const int c0 = c - c % a.chunk_len;
    const int w_lo = c0 - a.n_prev, w_hi = c0 + a.chunk_len;  // local window [w_lo, w_hi)
    const int64_t bh = (int64_t)b * a.H + h;
    {  // the pooled (mean) query of this query block
        __shared__ float part[SELECT_THREADS / (D / 8)][D];
        const uint16_t *frame = a.q + (int64_t)b * a.q_sb + (int64_t)h * a.q_sh + (int64_t)t * a.P * a.q_sr;
        // every row of the query block in one round of loads
        constexpr int UNROLL = QUERY_BLOCK / (SELECT_THREADS / (D / 8));
        pool_segment<D, UNROLL>(frame, a.q_sr, qi * QUERY_BLOCK, min(qi * QUERY_BLOCK + QUERY_BLOCK, a.P), part, qv);
    }
    for (int i = threadIdx.x; i < n_entries; i += SELECT_THREADS) flag[i] = 0;
    if (threadIdx.x == 0) {
        // history candidates in ascending order
        int n = 0;
        for (int f = 0; f < min(c0, a.T_kv); ++f)
            if (!(f < a.n_sink || (f >= w_lo && f < w_hi))) f_id[n++] = f;
        n_hist_s = n;
    }
    __syncthreads();
    const int n_hist = n_hist_s;
    // frame scores, four per warp at a time
    for (int i0 = 4 * warp; i0 < n_hist; i0 += 4 * nwarps) {
        const float *key[4];
        bool on[4];
        float sc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            on[u] = i0 + u < n_hist;
            key[u] = a.kf + (bh * a.T_kv + (on[u] ? f_id[i0 + u] : 0)) * D;
        }
        warp_dots<D, 4>(qv, key, on, sc);
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (on[u]) f_score[i0 + u] = sc[u];
        }
    }
    __syncthreads();
    // top k_frames: a candidate is kept when fewer than k_frames others rank before it
    for (int i = threadIdx.x; i < n_hist; i += SELECT_THREADS)
        f_taken[i] = rank_of(f_score, f_id, n_hist, f_score[i], f_id[i]) < a.k_frames ? 1 : 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0;
        for (int i = 0; i < n_hist; ++i)
            if (f_taken[i]) sel[n++] = f_id[i];
        n_sel_s = n;
    }
    __syncthreads();
    const int n_sel = n_sel_s;
    const int n_bc = n_sel * a.nblk;
    // block scores of the selected frames, four per warp at a time
    for (int i0 = 4 * warp; i0 < n_bc; i0 += 4 * nwarps) {
        const float *key[4];
        bool on[4];
        float sc[4];
        int ids[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u;
            on[u] = i < n_bc;
            const int f = on[u] ? sel[i / a.nblk] : 0, bb = on[u] ? i % a.nblk : 0;
            ids[u] = f * a.nblk + bb;
            key[u] = a.kb + ((bh * a.T_kv + f) * a.nblk + bb) * D;
        }
        warp_dots<D, 4>(qv, key, on, sc);
        if (lane == 0) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (on[u]) {
                    b_score[i0 + u] = sc[u];
                    b_id[i0 + u] = ids[u];
                }
        }
    }
    __syncthreads();
    // top k_blocks of the selected frames' blocks
    for (int i = threadIdx.x; i < n_bc; i += SELECT_THREADS)
        if (rank_of(b_score, b_id, n_bc, b_score[i], b_id[i]) < a.k_blocks) flag[b_id[i]] = 1;
    // always-attended frames: every block
    for (int i = threadIdx.x; i < n_entries; i += SELECT_THREADS) {
        const int f = i / a.nblk;
        if (f < a.n_sink || (f >= w_lo && f < w_hi)) flag[i] = 1;
    }
    __syncthreads();
    // compaction in id order: block-wide prefix count, SELECT_THREADS ids per round
    int32_t *out = a.blocks + (((bh * a.Tq + t) * a.nqb) + qi) * a.Amax;
    int base = 0;
    for (int r0 = 0; r0 < n_entries; r0 += SELECT_THREADS) {
        const int i = r0 + threadIdx.x;
        const bool on = i < n_entries && flag[i];
        const unsigned m = __ballot_sync(0xffffffffu, on);
        if (lane == 0) warp_tot[warp] = __popc(m);
        __syncthreads();
        int before = base;
        for (int w = 0; w < warp; ++w) before += warp_tot[w];
        before += __popc(m & ((1u << lane) - 1u));
        if (on && before < a.Amax) out[before] = i;
        int total = 0;
        for (int w = 0; w < nwarps; ++w) total += warp_tot[w];
        base += total;
        __syncthreads();
    }
    for (int i = base + threadIdx.x; i < a.Amax; i += SELECT_THREADS) out[i] = -1;
    if (threadIdx.x == 0) a.counts[((bh * a.Tq + t) * a.nqb) + qi] = min(base, a.Amax);
}

bool params_ok(const sfa_set_params *p, int P, int k_frames, int k_blocks)
{
    if (!p || P < 1 || k_frames < 0 || k_blocks < 0) return false;
    if (p->T_kv < 1 || p->Tq < 1 || p->q_off < 0 || (int64_t)p->q_off + p->Tq > p->T_kv) return false;
    if (p->n_sink < 0 || p->n_prev < 0 || p->chunk_len < 1) return false;
    const int64_t nblk = (P + KEY_BLOCK - 1) / KEY_BLOCK;
    return (int64_t)p->T_kv * nblk <= MAX_ENTRIES;
}

int64_t max_count(const sfa_set_params *p, int P, int k_frames, int k_blocks)
{
    const int64_t nblk = (P + KEY_BLOCK - 1) / KEY_BLOCK;
    const int64_t always = std::min<int64_t>((int64_t)p->n_sink + p->n_prev + p->chunk_len, p->T_kv) * nblk;
    return always + std::min<int64_t>(k_blocks, (int64_t)k_frames * nblk);
}

struct WsLayout {
    size_t kf, kb, qb, total;
};

WsLayout ws_layout(const sfa_attn_desc *d)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t nblk = (d->P + KEY_BLOCK - 1) / KEY_BLOCK, nqb = (d->P + QUERY_BLOCK - 1) / QUERY_BLOCK;
    const size_t bh = (size_t)d->B * d->H;
    WsLayout w;
    w.kf = 0;
    w.kb = up(bh * d->T_kv * d->d * 4);
    w.qb = w.kb + up(bh * d->T_kv * nblk * d->d * 4);
    w.total = w.qb + up(bh * d->Tq * nqb * d->d * 4);
    return w;
}

bool desc_ok(const sfa_attn_desc *d)
{
    if (!d || d->B < 0 || d->H < 1 || d->Tq < 1 || d->T_kv < 1 || d->P < 1 || d->Amax < 1) return false;
    if ((int64_t)d->Tq * d->P >= ((int64_t)1 << 31) || (int64_t)d->T_kv * d->P >= ((int64_t)1 << 31)) return false;
    if ((int64_t)d->B * d->H > 65535 || d->T_kv > 65535) return false;  // grid y of the pooling launch; frame ids
    return true;
}

bool stride_ok(const int64_t *s, int d)
{
    return s[2] >= d && s[0] >= 0 && s[1] >= 0 && s[0] % 8 == 0 && s[1] % 8 == 0 && s[2] % 8 == 0;
}

// Pooling launch: the keys (with their frame means) and/or the queries of a descriptor.
template <int D>
sfa_status run_pool(const sfa_attn_desc *d, const void *q, const void *k, uint8_t *ws, bool keys, bool queries,
                    cudaStream_t s)
{
    const WsLayout w = ws_layout(d);
    float *kf = reinterpret_cast<float *>(ws + w.kf), *kb = reinterpret_cast<float *>(ws + w.kb);
    float *qb = reinterpret_cast<float *>(ws + w.qb);
    const int nblk = (d->P + KEY_BLOCK - 1) / KEY_BLOCK, nqb = (d->P + QUERY_BLOCK - 1) / QUERY_BLOCK;
    const unsigned bh = (unsigned)d->B * d->H;
    PoolArgs pa;
    pa.k = static_cast<const uint16_t *>(k);
    pa.q = static_cast<const uint16_t *>(q);
    pa.k_sb = d->k_stride[0];
    pa.k_sh = d->k_stride[1];
    pa.k_sr = d->k_stride[2];
    pa.q_sb = d->q_stride[0];
    pa.q_sh = d->q_stride[1];
    pa.q_sr = d->q_stride[2];
    pa.H = d->H;
    pa.P = d->P;
    pa.T_kv = d->T_kv;
    pa.Tq = d->Tq;
    pa.nblk = nblk;
    pa.nqb = nqb;
    pa.k_on = keys ? 1 : 0;
    pa.kb = kb;
    pa.qb = qb;
    const unsigned grid_x = (unsigned)((keys ? nblk * d->T_kv : 0) + (queries ? nqb * d->Tq : 0));
    hsa_pool_kernel<D><<<dim3(grid_x, bh), POOL_THREADS, 0, s>>>(pa);
    if (keys) {
        const int64_t n_kf = (int64_t)bh * d->T_kv * D;
        hsa_frame_mean_kernel<D><<<(unsigned)((n_kf + 255) / 256), 256, 0, s>>>(kb, n_kf, d->P, nblk, kf);
    }
    return launch_status();
}

// Selection from the pooled keys and queries in the workspace.
template <int D>
sfa_status run_select(const sfa_attn_desc *d, const sfa_set_params *p, int k_frames, int k_blocks, const void *q,
                      uint8_t *ws, int32_t *blocks, int32_t *counts, cudaStream_t s)
{
    const WsLayout w = ws_layout(d);
    SelectArgs a;
    a.B = d->B;
    a.H = d->H;
    a.Tq = d->Tq;
    a.T_kv = d->T_kv;
    a.P = d->P;
    a.nblk = (d->P + KEY_BLOCK - 1) / KEY_BLOCK;
    a.nqb = (d->P + QUERY_BLOCK - 1) / QUERY_BLOCK;
    a.Amax = d->Amax;
    a.q_off = p->q_off;
    a.n_sink = p->n_sink;
    a.n_prev = p->n_prev;
    a.chunk_len = p->chunk_len;
    a.k_frames = k_frames;
    a.k_blocks = k_blocks;
    a.kf = reinterpret_cast<const float *>(ws + w.kf);
    a.kb = reinterpret_cast<const float *>(ws + w.kb);
    a.q = static_cast<const uint16_t *>(q);
    a.q_sb = d->q_stride[0];
    a.q_sh = d->q_stride[1];
    a.q_sr = d->q_stride[2];
    a.blocks = blocks;
    a.counts = counts;
    const int n_sel_max = std::min(k_frames, d->T_kv);
    const size_t n_bc_max = (size_t)n_sel_max * a.nblk;
    const size_t smem = (size_t)d->T_kv * 8 + n_bc_max * 8 + (size_t)n_sel_max * 4 + d->T_kv +
                        (size_t)d->T_kv * a.nblk;
    if (smem > 200 * 1024) return SFA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(hsa_select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return SFA_ERR_CUDA;
    const int64_t grid = (int64_t)d->B * d->H * d->Tq * a.nqb;
    hsa_select_kernel<D><<<(unsigned)grid, SELECT_THREADS, smem, s>>>(a);
    return launch_status();
}

// Common host checks of the selection entry points (the tensors present are checked).
sfa_status select_checks(const sfa_attn_desc *d, const sfa_set_params *p, int k_frames, int k_blocks, const void *q,
                         const void *k, void *workspace, size_t workspace_bytes, const int32_t *blocks,
                         const int32_t *counts, bool need_k)
{
    if (!desc_ok(d) || !params_ok(p, d ? d->P : 0, k_frames, k_blocks)) return SFA_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return SFA_ERR_UNSUPPORTED;
    if (p->T_kv != d->T_kv || p->Tq != d->Tq) return SFA_ERR_INVALID_ARG;
    if (max_count(p, d->P, k_frames, k_blocks) > d->Amax) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!q || (need_k && !k) || !workspace || !blocks || !counts) return SFA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(q) % 16 || (need_k && reinterpret_cast<uintptr_t>(k) % 16) ||
        reinterpret_cast<uintptr_t>(workspace) % 256)
        return SFA_ERR_INVALID_ARG;
    if (!stride_ok(d->q_stride, d->d) || (need_k && !stride_ok(d->k_stride, d->d))) return SFA_ERR_INVALID_ARG;
    if (workspace_bytes < ws_layout(d).total) return SFA_ERR_INVALID_ARG;
    return SFA_OK;
}

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_hsa_max_count(const sfa_set_params *p, int32_t P, int32_t k_frames, int32_t k_blocks,
                                        int32_t *amax_out)
{
    if (!amax_out || !params_ok(p, P, k_frames, k_blocks)) return SFA_ERR_INVALID_ARG;
    const int64_t m = max_count(p, P, k_frames, k_blocks);
    if (m > INT32_MAX) return SFA_ERR_INVALID_ARG;
    *amax_out = (int32_t)std::max<int64_t>(m, 1);
    return SFA_OK;
}

extern "C" sfa_status sfa_hsa_workspace(const sfa_attn_desc *d, size_t *bytes)
{
    if (!bytes || !desc_ok(d)) return SFA_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return SFA_ERR_UNSUPPORTED;
    *bytes = ws_layout(d).total;
    return SFA_OK;
}

extern "C" sfa_status sfa_hsa_select(const sfa_attn_desc *d, const sfa_set_params *p, int32_t k_frames,
                                     int32_t k_blocks, const void *q, const void *k, void *workspace,
                                     size_t workspace_bytes, int32_t *blocks, int32_t *counts, sfa_stream_t stream)
{
    sfa_status st = select_checks(d, p, k_frames, k_blocks, q, k, workspace, workspace_bytes, blocks, counts, true);
    if (st != SFA_OK || d->B == 0) return st;
    cudaStream_t s = as_cuda(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    st = d->d == 128 ? run_pool<128>(d, q, k, ws, true, false, s) : run_pool<64>(d, q, k, ws, true, false, s);
    if (st != SFA_OK) return st;
    return d->d == 128 ? run_select<128>(d, p, k_frames, k_blocks, q, ws, blocks, counts, s)
                       : run_select<64>(d, p, k_frames, k_blocks, q, ws, blocks, counts, s);
}

extern "C" sfa_status sfa_hsa_pool_keys(const sfa_attn_desc *d, const void *k, void *workspace,
                                        size_t workspace_bytes, sfa_stream_t stream)
{
    if (!desc_ok(d)) return SFA_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return SFA_ERR_UNSUPPORTED;
    if ((int64_t)d->T_kv * ((d->P + KEY_BLOCK - 1) / KEY_BLOCK) > MAX_ENTRIES) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!k || !workspace || reinterpret_cast<uintptr_t>(k) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256)
        return SFA_ERR_INVALID_ARG;
    if (!stride_ok(d->k_stride, d->d) || workspace_bytes < ws_layout(d).total) return SFA_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    return d->d == 128 ? run_pool<128>(d, nullptr, k, ws, true, false, s)
                       : run_pool<64>(d, nullptr, k, ws, true, false, s);
}

extern "C" sfa_status sfa_hsa_select_pooled(const sfa_attn_desc *d, const sfa_set_params *p, int32_t k_frames,
                                            int32_t k_blocks, const void *q, void *workspace, size_t workspace_bytes,
                                            int32_t *blocks, int32_t *counts, sfa_stream_t stream)
{
    sfa_status st =
        select_checks(d, p, k_frames, k_blocks, q, nullptr, workspace, workspace_bytes, blocks, counts, false);
    if (st != SFA_OK || d->B == 0) return st;
    cudaStream_t s = as_cuda(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    return d->d == 128 ? run_select<128>(d, p, k_frames, k_blocks, q, ws, blocks, counts, s)
                       : run_select<64>(d, p, k_frames, k_blocks, q, ws, blocks, counts, s);
}
