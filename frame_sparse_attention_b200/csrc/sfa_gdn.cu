// ARL2 inter-frame branch: gated delta rule with frame-level state access, sm_100a.
//
// "Resumen Técnico: Asistir Localmente, Recordar Linealmente (ARL2)", §2.1 (Rama
// Inter-Cuadro): a fixed-size state S [d x d] per (batch, head) replaces the KV cache;
// frame N reads it as O_N = Q'_N S_{N-1} and then updates it as
//   S_N = alpha_N S_{N-1} + K'_N^T diag(beta_N) (V'_N - K'_N S_{N-1});
// §2.2: every token of a frame reads the same pre-update state (frame-level access), and
// intermediate denoising steps read without writing (update = 0).
//
// The update is linear in the state:
//   S_N = alpha_N S_{N-1} - M_N S_{N-1} + B_N,   M_N = K^T diag(beta) K,  B_N = K^T diag(beta) V,
// and M_N, B_N (d x d each) depend on frame N's tokens only.  So the work splits in two:
//   gdn_prep_kernel: one CTA per (batch, head, frame) forms M_N (bf16) and B_N (fp32) on
//     the tensor cores, all frames at once (K~ = sqrt(beta) K and V~ = sqrt(beta) V are
//     formed in shared memory, then M_N = K~^T K~ and B_N = K~^T V~);
//   gdn_kernel: G CTAs per (batch, head) each run the recurrence over the frames (one
//     128 x 128 x 128 product M_N S_{N-1} per frame, the rest in fp32), and each computes
//     O = Q S_{N-1} for its own token tiles of every frame (in frame n, CTA g takes the
//     tiles i with (i + n) mod G = g).  The G CTAs of a head repeat the same small
//     recurrence and never wait for one another.
// Read-only steps (update = 0) run only the O contraction with the input state.
// In both kernels warps 0-7 (two threads per TMEM lane, 64 columns each) do the
// element-wise work.  In gdn_prep_kernel warp 8 issues the TMA copies and the MMAs; in
// gdn_kernel warp 8 issues the MMAs and warp 9 the TMA copies, so that no copy waits in
// the issue stream of the frame's recurrence.  Every wait is bounded; a wait that runs
// out stores SFA_ERR_TIMEOUT and the CTA drains and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sfa.h"
#include "sfa_internal.h"
#include "sfa_ptx.cuh"

namespace sfa {
namespace {

constexpr int GD = 128;          // d_k = d_v
constexpr int GBM = 128;         // tokens per tile
constexpr int GEPI = 256;        // warps 0-7: element-wise work (two threads per TMEM lane)
constexpr int GW_MMA = 8;        // warp 8: TMA copies and MMAs (gdn_prep_kernel), MMAs (gdn_kernel)
constexpr int GW_TMA = 9;        // warp 9 of gdn_kernel: its TMA copies
constexpr int GTHREADS = GEPI + 32;       // gdn_prep_kernel
constexpr int GTHREADS_REC = GEPI + 64;   // gdn_kernel
constexpr int G_BOX = 128 * 128; // one 128-row x 64-column bf16 box (128-byte swizzle)
constexpr int G_TILE = 2 * G_BOX;

// gdn_prep_kernel shared memory: three stages of 64-token K, V tiles (scaled in place);
// two CTAs share an SM, so one streams its tiles while the other starts or ends a frame
constexpr int PBM = 64;                  // tokens per prep tile
constexpr int P_BOX = PBM * 128;         // one 64-row x 64-column bf16 box (128-byte swizzle)
constexpr int P_TILE = 2 * P_BOX;        // one K or V tile
constexpr int PR_STAGES = 3, PR_SLOT = 2 * P_TILE;
constexpr int PR_BAR = PR_STAGES * PR_SLOT;
constexpr int PR_SMEM = PR_BAR + 256 + 1024;
static_assert(PR_STAGES * PR_SLOT >= G_TILE, "the stages hold the bf16 M_N tile for its store");
constexpr uint32_t PT_M = 0, PT_B = 128;  // tensor-memory columns (256 allocated)

// gdn_kernel shared memory: the bf16 state (B operand), two M_N tiles, a ring of Q tiles
// (each Q buffer then stages its tile's O for the TMA store)
constexpr int NQ = 4;
constexpr int MS_S = 0, MS_M = G_TILE, MS_Q = 3 * G_TILE;
constexpr int MS_BAR = MS_Q + NQ * G_TILE;
constexpr int MS_SMEM = MS_BAR + 256 + 1024;
constexpr uint32_t T_D = 0, T_O0 = 128, T_SST = 384;  // tensor memory: M S, two O buffers, fp32 state

struct GdnArgs {
    int32_t B, H, T, P, n_tiles, update;
    int32_t G;           // CTAs per (batch, head) in gdn_kernel
    const float *alpha;  // [B][H][T]
    const float *beta;   // [B][H][T*P]
    const float *s_in;   // [B][H][d][d] or null (zeros)
    float *s_out;        // [B][H][d][d]
    const float *bws;    // fp32 B_N, written by gdn_prep_kernel: per (b, h, frame) [32][d][4], element
                         // (row r, column 4 cg + i) at cg * 4 d + 4 r + i, so that the 16-byte
                         // pieces of 32 consecutive rows lie side by side
    int32_t *status;
    uint64_t timeout_ns;
    uint32_t debug_flags;  // SFA_DEBUG_STALL_GDN_STATE: the input state is never signalled ready
};

__device__ __forceinline__ uint64_t gns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bounded wait; false (and the abort flag set, status written) when it runs out.  Inline
// throughout: a call would make the thread first wait for the loads it has in flight.
__device__ __forceinline__ bool gwait_slow(uint32_t bar, uint32_t parity, volatile int32_t *abort, int32_t *status,
                                           uint64_t limit)
{
    const uint64_t t0 = gns();
    for (uint32_t spins = 1;; ++spins) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if ((spins & 63) == 0 && (gns() - t0 > limit || spins > (1u << 30))) {
            *abort = 1;
            if (status) atomicCAS(status, 0, SFA_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool gwait(uint32_t bar, uint32_t parity, volatile int32_t *abort, int32_t *status,
                                      uint64_t limit)
{
    return mbar_try_wait(bar, parity) || gwait_slow(bar, parity, abort, status, limit);
}

// wait for copies already in flight, whatever the abort flag says, for at most 2 s
__device__ __forceinline__ void gdrain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = gns();
    while (!mbar_try_wait(bar, parity) && gns() - t0 < 2000000000ull) {
    }
}

__device__ __forceinline__ uint32_t swz(int row, int col)  // byte offset of bf16 (row, col) in a swizzled tile
{
    const int box = col >> 6, chunk = (col & 63) >> 3;
    return (uint32_t)(box * G_BOX + row * 128 + ((chunk ^ (row & 7)) << 4) + (col & 7) * 2);
}

// byte offset of 16-byte chunk `chunk` (0-7) of row `row` of box `box` in a swizzled
// 64-row prep tile
__device__ __forceinline__ uint32_t pswz(int box, int row, int chunk)
{
    return (uint32_t)(box * P_BOX + row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ float bf16f(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

// x * s for the 8 bf16 of a 16-byte chunk, rounded back to bf16
__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float s)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        o[j] = pack_bf16x2(s * bf16f((uint16_t)(w[j] & 0xffffu)), s * bf16f((uint16_t)(w[j] >> 16)));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------------------------
// M_N = K^T diag(beta) K (bf16, the A operand of the recurrence) and B_N = K^T diag(beta) V
// (fp32) of one frame: K~ = sqrt(beta) K and V~ = sqrt(beta) V are formed in place, then
// M_N = K~^T K~ and B_N = K~^T V~ accumulate over the frame's tiles (M = N = d, K = 64
// tokens per tile; both operands MN-major).  beta must be >= 0 (a step size); a negative or
// NaN beta stores SFA_ERR_INVALID_ARG and its token is left out.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(GTHREADS, 2)
    gdn_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_mw, const __grid_constant__ GdnArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem), bb = sbase + PR_BAR;
    auto kv_full = [&](int s) { return bb + 8 * s; };        // K, V of stage s landed
    auto scaled = [&](int s) { return bb + 48 + 8 * s; };    // K~, V~ of stage s formed (all threads)
    auto mma_done = [&](int s) { return bb + 96 + 8 * s; };  // the MMAs reading stage s are done
    const uint32_t fin = bb + 144, staged = bb + 152, drain = bb + 160;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PR_BAR + 176);
    volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(smem + PR_BAR + 180);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int fr = blockIdx.x;  // (b * H + h) * T + n
    const int bhi = fr / a.T, n = fr % a.T, b = bhi / a.H, h = bhi % a.H;
    const int nt = (a.P + PBM - 1) / PBM;  // 64-token tiles of the frame

    if (threadIdx.x == 0) {
        for (int s = 0; s < PR_STAGES; ++s) {
            mbar_init(kv_full(s), 1);
            mbar_init(scaled(s), GEPI);
            mbar_init(mma_done(s), 1);
        }
        mbar_init(fin, 1);
        mbar_init(staged, GEPI);
        mbar_init(drain, 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == GW_MMA) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_mw);
        }
        tmem_alloc(smem_u32(tmem_slot), 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the recurrence kernel may take the SMs this grid leaves free and set itself up; it
    // waits for this grid's results before it reads them
    pdl_launch_dependents();

    if (warp == GW_MMA) {
        constexpr uint32_t id_mm = idesc_bf16_f32(GD, GD, true) | (1u << 15);  // A and B MN-major
        int n_loaded = 0, n_seen = 0;  // tiles whose copies were issued / seen formed
        bool ok = true, issued = false;
        auto load = [&](int t) {
            const int s = t % PR_STAGES;
            const uint32_t dst = sbase + s * PR_SLOT;
            if (elect_one()) {
                mbar_arrive_expect_tx(kv_full(s), 2 * P_TILE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_load_5d(dst + kb * P_BOX, &tm_k, kv_full(s), kb * 64, t * PBM, n, h, b);
                    tma_load_5d(dst + P_TILE + kb * P_BOX, &tm_v, kv_full(s), kb * 64, t * PBM, n, h, b);
                }
            }
            __syncwarp();
            n_loaded = t + 1;
        };
        for (int t = 0; t < PR_STAGES && t < nt; ++t) load(t);
        for (int i = 0; i < nt && ok; ++i) {
            const int s = i % PR_STAGES;
            if (!(ok = __all_sync(0xffffffffu, gwait(scaled(s), (i / PR_STAGES) & 1, abort, a.status, a.timeout_ns))))
                break;
            n_seen = i + 1;
            tc_fence_after();
            const uint64_t dk = sdesc_sw128(sbase + s * PR_SLOT, P_BOX, 1024);           // K~ [tokens][d]
            const uint64_t dv = sdesc_sw128(sbase + s * PR_SLOT + P_TILE, P_BOX, 1024);  // V~ [tokens][d]
            if (elect_one()) {
#pragma unroll
                for (uint32_t kk = 0; kk < PBM / 16; ++kk) {
                    const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
                    mma_ss(tmem + PT_M, dk + ((kk * 2048) >> 4), dk + ((kk * 2048) >> 4), id_mm, acc);
                    mma_ss(tmem + PT_B, dk + ((kk * 2048) >> 4), dv + ((kk * 2048) >> 4), id_mm, acc);
                }
                tc_commit(mma_done(s));
            }
            __syncwarp();
            issued = true;
            // tile i + PR_STAGES - 1 takes the stage of tile i - 1 once that tile's MMAs are done
            if (i >= 1 && i + PR_STAGES - 1 < nt) {
                const int p = i - 1;
                if (!(ok = __all_sync(0xffffffffu, gwait(mma_done(p % PR_STAGES), (p / PR_STAGES) & 1, abort,
                                                          a.status, a.timeout_ns))))
                    break;
                load(i + PR_STAGES - 1);
            }
        }
        if (ok && nt > 0) {
            if (elect_one()) tc_commit(fin);
            __syncwarp();
        }
        if (__any_sync(0xffffffffu, *abort != 0)) {
            if (issued) {  // tensor cores idle before TMEM is freed
                if (elect_one()) tc_commit(drain);
                __syncwarp();
                gdrain(drain, 0);
            }
            for (int t = n_seen; t < n_loaded; ++t) gdrain(kv_full(t % PR_STAGES), (t / PR_STAGES) & 1);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------- tile row tr, columns 32 cq .. + 31
        const int e = threadIdx.x, qd = warp & 3, hc = warp >> 2;
        const int r = qd * 32 + lane, c0 = hc * 2;  // TMEM lane and column half of the epilogue
        const int tr = (warp & 1) * 32 + lane, cq = warp >> 1;
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        const float *beta = a.beta + (int64_t)fr * a.P;
        bool ok = true;
        float bt_next = tr < a.P ? beta[tr] : 0.f;
        for (int i = 0; i < nt; ++i) {
            const int s = i % PR_STAGES, row = i * PBM + tr;
            const float bt = bt_next;
            bt_next = (i + 1 < nt && row + PBM < a.P) ? beta[row + PBM] : 0.f;
            if (!(ok = __all_sync(0xffffffffu, gwait(kv_full(s), (i / PR_STAGES) & 1, abort, a.status, a.timeout_ns))))
                break;
            float sb = 0.f;
            if (row < a.P) {
                if (bt >= 0.f)
                    sb = sqrtf(bt);
                else if (a.status)
                    atomicCAS(a.status, 0, SFA_ERR_INVALID_ARG);
            }
            // K~ and V~ of tile row tr, columns 32 cq .. 32 cq + 31, in place
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint32_t off = s * PR_SLOT + pswz(cq >> 1, tr, (cq & 1) * 4 + q);
                uint4 *pk = reinterpret_cast<uint4 *>(smem + off), *pv = reinterpret_cast<uint4 *>(smem + off + P_TILE);
                *pk = scale_bf16x8(*pk, sb);
                *pv = scale_bf16x8(*pv, sb);
            }
            fence_proxy_async_smem();
            mbar_arrive(scaled(s));
        }
        if (ok && nt > 0 && (ok = __all_sync(0xffffffffu, gwait(fin, 0, abort, a.status, a.timeout_ns)))) {
            tc_fence_after();
            // M_N row r as bf16 into stage 0 (the layout of the bf16 map's two boxes; every
            // stage is free now); B_N row r straight to global memory, 16 bytes per store, the
            // lanes of a warp (32 consecutive rows) writing 512 contiguous bytes
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = c0 + cc;
                uint32_t m[32], bv[32];
                tmem_ld32(lane_base + PT_M + c * 32, m);
                tmem_ld32(lane_base + PT_B + c * 32, bv);
                tmem_wait_ld_regs(m);
                tmem_wait_ld_regs(bv);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        w[j] = pack_bf16x2(__uint_as_float(m[8 * q + 2 * j]), __uint_as_float(m[8 * q + 2 * j + 1]));
                    st_shared_v4(sbase + swz(r, c * 32 + q * 8), w);
                }
                float4 *bo = reinterpret_cast<float4 *>(const_cast<float *>(a.bws)) + ((int64_t)fr * 32 + c * 8) * GD + r;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    __stcg(bo + j * GD, make_float4(__uint_as_float(bv[4 * j]), __uint_as_float(bv[4 * j + 1]),
                                                    __uint_as_float(bv[4 * j + 2]), __uint_as_float(bv[4 * j + 3])));
            }
            fence_proxy_async_smem();
            mbar_arrive(staged);
            if (e == 0 && gwait(staged, 0, abort, a.status, a.timeout_ns)) {
                const int y = fr * GD;
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) tma_store_2d(&tm_mw, sbase + kb * G_BOX, kb * 64, y);
                bulk_commit_and_wait_all();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == GW_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------------------------
// The recurrence and O = Q S_{N-1}: CTA g of a (batch, head) runs
//   S_N = alpha_N S_{N-1} - M_N bf16(S_{N-1}) + B_N   (fp32 state in TMEM)
// frame by frame (M_N S as one 128 x 128 x 128 MMA), and the O MMAs of its tiles of frame N
// read the same bf16(S_{N-1}) in shared memory; the state buffer is rewritten once they are
// done.  Tiles of consecutive frames stream through a ring of NQ Q buffers; O is read out
// of one of two TMEM buffers, staged in the tile's Q buffer and written by a TMA store
// that warp 9 issues, which then refills the buffer with the tile NQ places further on.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(GTHREADS_REC, 1)
    gdn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ CUtensorMap tm_mw, const __grid_constant__ GdnArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem), bb = sbase + MS_BAR;
    auto q_full = [&](int s) { return bb + 8 * s; };         // Q of ring slot s landed
    auto m_full = [&](int s) { return bb + 32 + 8 * s; };    // M_N of slot s landed
    const uint32_t d_done = bb + 48;                         // M_N S in TMEM
    const uint32_t s_free = bb + 56;                         // the frame's MMAs no longer read S
    auto o_done = [&](int u) { return bb + 64 + 8 * u; };    // O of a tile in TMEM buffer u
    // O of the tile in Q buffer s read out of TMEM and staged in that buffer (all).  One
    // barrier per Q buffer rather than per TMEM buffer: the TMA warp waits for the tiles in
    // order to send them, and the next completion of a Q buffer's barrier needs the copy the
    // TMA warp makes only after that wait (no phase can be skipped unseen)
    auto o_staged = [&](int s) { return bb + 112 + 8 * s; };
    auto m_free = [&](int s) { return bb + 144 + 8 * s; };  // the product reading M slot s is done
    const uint32_t s_ready = bb + 96;                        // state of the next frame written (all)
    const uint32_t drain = bb + 104;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + MS_BAR + 160);
    volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(smem + MS_BAR + 164);
    int32_t *landed = reinterpret_cast<int32_t *>(smem + MS_BAR + 168);  // Q tiles, M frames the MMA warp saw land
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / a.G, g = blockIdx.x % a.G, b = bh / a.H, h = bh % a.H;
    const bool upd = a.update != 0;
    // Tiles of frame n that this CTA takes: first(n), first(n) + G, ...  The assignment
    // rotates by one CTA per frame, so that when the tiles of a frame do not divide evenly
    // among the G CTAs the extra ones fall on a different CTA in every frame: each CTA then
    // carries its share of them instead of CTA 0 carrying all of them in every frame (every
    // CTA runs the whole recurrence, so the slowest one sets the call's time).
    auto first_tile = [&](int n) { return (g - n % a.G + a.G) % a.G; };
    auto tiles_in = [&](int n) { return (a.n_tiles - first_tile(n) + a.G - 1) / a.G; };

    if (threadIdx.x == 0) {
        const uint32_t single[10] = {q_full(0), q_full(1), q_full(2), q_full(3), m_full(0),
                                     m_full(1), d_done,    s_free,    o_done(0), o_done(1)};
        for (uint32_t x : single) mbar_init(x, 1);
        mbar_init(drain, 1);
        for (int x = 0; x < NQ; ++x) mbar_init(o_staged(x), GEPI);
        mbar_init(m_free(0), 1);
        mbar_init(m_free(1), 1);
        mbar_init(s_ready, GEPI);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == GW_MMA) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_o);
            if (upd) tma_prefetch_desc(&tm_mw);
        }
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int q_loaded = 0, m_loaded = 0;  // copies the TMA warp issued

    if (warp == GW_MMA) {
        // ---------------------------------------------------------------- MMA
        const uint64_t ds = sdesc_sw128(sbase + MS_S, G_BOX, 1024);  // S: [d_k rows][d_v], MN-major B
        constexpr uint32_t id_qs = idesc_bf16_f32(GBM, GD, true);
        int q_landed = 0, m_landed = 0;
        bool ok = true, issued = false;
        int it = 0;
        for (int n = 0; n < a.T && ok; ++n) {
            if ((upd || n == 0) &&
                !(ok = __all_sync(0xffffffffu, gwait(s_ready, n & 1, abort, a.status, a.timeout_ns))))
                break;
            if (upd) {
                if (!(ok = __all_sync(0xffffffffu, gwait(m_full(n & 1), (n >> 1) & 1, abort, a.status, a.timeout_ns))))
                    break;
                m_landed = n + 1;
                tc_fence_after();
                const uint64_t dm = sdesc_sw128(sbase + MS_M + (n & 1) * G_TILE, 16, 1024);  // M_N, K-major A
                if (elect_one()) {
#pragma unroll
                    for (uint32_t kk = 0; kk < GD / 16; ++kk) {
                        const uint32_t ka = (kk >> 2) * G_BOX + (kk & 3) * 32;
                        mma_ss(tmem + T_D, dm + (ka >> 4), ds + ((kk * 2048) >> 4), id_qs, kk > 0);
                    }
                    tc_commit(d_done);
                    tc_commit(m_free(n & 1));
                }
                __syncwarp();
                issued = true;
            }
            const int per = tiles_in(n);
            for (int ii = 0; ii < per && ok; ++ii, ++it) {
                const int s = it % NQ, u = it & 1;
                if (!(ok = __all_sync(0xffffffffu, gwait(q_full(s), (it / NQ) & 1, abort, a.status, a.timeout_ns))))
                    break;
                q_landed = it + 1;
                // TMEM buffer u last held tile it - 2: read out and staged
                if (it >= 2 && !(ok = __all_sync(0xffffffffu, gwait(o_staged((it - 2) % NQ), ((it - 2) / NQ) & 1, abort,
                                                                      a.status, a.timeout_ns))))
                    break;
                tc_fence_after();
                const uint64_t dq = sdesc_sw128(sbase + MS_Q + s * G_TILE, 16, 1024);  // Q tile, K-major A
                if (elect_one()) {
#pragma unroll
                    for (uint32_t kk = 0; kk < GD / 16; ++kk) {
                        const uint32_t ka = (kk >> 2) * G_BOX + (kk & 3) * 32;
                        mma_ss(tmem + T_O0 + u * 128, dq + (ka >> 4), ds + ((kk * 2048) >> 4), id_qs, kk > 0);
                    }
                    tc_commit(o_done(u));
                    // after the frame's last MMA that reads S: the state may be rewritten
                    if (ii == per - 1) tc_commit(s_free);
                }
                __syncwarp();
                issued = true;
            }
        }
        if (__any_sync(0xffffffffu, *abort != 0) && issued) {  // tensor cores idle before TMEM is freed
            if (elect_one()) tc_commit(drain);
            __syncwarp();
            gdrain(drain, 0);
        }
        if (lane == 0) {
            landed[0] = q_landed;
            landed[1] = m_landed;
        }
        __syncwarp();
    } else if (warp == GW_TMA) {
        // ---------------------------------------------------------------- TMA: Q, M_N in, O out
        int total = 0;
        for (int n = 0; n < a.T; ++n) total += tiles_in(n);
        bool ok = true;
        // the CTA's tiles in order (frame n, j-th tile of the frame), one cursor for the Q
        // loads and one for the O stores, each visiting them once in that order
        struct Cursor {
            int n, j;
        };
        Cursor lc = {0, 0}, sc = {0, 0};
        auto next_tile = [&](Cursor &c, int &n, int &i) {
            n = c.n;
            i = first_tile(c.n) + c.j * a.G;
            if (++c.j == tiles_in(c.n)) {
                c.j = 0;
                ++c.n;
            }
        };
        auto load_q = [&](int t) {  // tile t of the CTA's sequence, the next one the cursor gives
            int n, i;
            next_tile(lc, n, i);
            const int s = t % NQ;
            if (elect_one()) {
                mbar_arrive_expect_tx(q_full(s), G_TILE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
                    tma_load_5d(sbase + MS_Q + s * G_TILE + kb * G_BOX, &tm_q, q_full(s), kb * 64, i * GBM, n, h, b);
            }
            __syncwarp();
        };
        auto load_m = [&](int n) {
            const int s = n & 1, y = (bh * a.T + n) * GD;
            if (elect_one()) {
                mbar_arrive_expect_tx(m_full(s), G_TILE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
                    tma_load_2d(sbase + MS_M + s * G_TILE + kb * G_BOX, &tm_mw, m_full(s), kb * 64, y);
            }
            __syncwarp();
        };
        // O of tile t (staged by the epilogue in its Q buffer) -> global; lane 0 owns the
        // bulk groups
        auto store_o = [&](int t) {
            int n, i;
            next_tile(sc, n, i);
            const uint32_t src = sbase + MS_Q + (t % NQ) * G_TILE;
            if (lane == 0) {
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) tma_store_5d(&tm_o, src + kb * G_BOX, kb * 64, i * GBM, n, h, b);
                tma_store_commit();
            }
            __syncwarp();
        };
        for (; q_loaded < NQ && q_loaded < total; ++q_loaded) load_q(q_loaded);
        pdl_wait();  // M_N comes from the preparation kernel
        if (upd)
            for (; m_loaded < 2 && m_loaded < a.T; ++m_loaded) load_m(m_loaded);
        int t = 0;
        for (int n = 0; n < a.T && ok; ++n) {
            if (upd && n + 2 < a.T) {  // M_{n+2} takes the slot of M_n once the product of frame n is done
                if (!(ok = __all_sync(0xffffffffu, gwait(m_free(n & 1), (n >> 1) & 1, abort, a.status, a.timeout_ns))))
                    break;
                load_m(n + 2);
                m_loaded = n + 3;
            }
            const int per = tiles_in(n);
            // the O stores of frame n wait for the product of frame n + 1 to be done, so that
            // their shared-memory reads do not slow it down (it sets the pace of the frames);
            // not when a Q buffer must be refilled within the frame (the frame's products
            // would wait for a store that waits for the next frame)
            if (upd && n + 1 < a.T && per <= NQ &&
                !(ok = __all_sync(0xffffffffu, gwait(m_free((n + 1) & 1), ((n + 1) >> 1) & 1, abort, a.status,
                                                     a.timeout_ns))))
                break;
            for (int ii = 0; ii < per && ok; ++ii, ++t) {
                // tile t's O staged in its Q buffer: send it; the buffer then takes tile t + NQ
                if (!(ok = __all_sync(0xffffffffu, gwait(o_staged(t % NQ), (t / NQ) & 1, abort, a.status, a.timeout_ns))))
                    break;
                store_o(t);
                if (t + NQ < total) {
                    if (lane == 0) tma_store_wait_read_all();
                    __syncwarp();
                    load_q(t + NQ);
                    q_loaded = t + NQ + 1;
                }
            }
        }
        if (lane == 0) bulk_commit_and_wait_all();  // every O store complete
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- row r, half hc
        // warps w and w + 4 share TMEM lanes 32 (w mod 4) .. + 31 (tile rows, state rows) and
        // take 64 columns each
        const int qd = warp & 3, hc = warp >> 2;
        const int r = qd * 32 + lane;  // TMEM lane = tile row = state row (d_k index)
        const int c0 = hc * 2;         // this thread's 32-column chunks: c0, c0 + 1
        const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
        const int64_t bhi = (int64_t)b * a.H + h;
        // state in: fp32 row r into TMEM, bf16 row r into the B-operand tile (this half)
        {
            float srow[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) srow[c] = a.s_in ? a.s_in[(bhi * GD + r) * GD + hc * 64 + c] : 0.f;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(srow[cc * 32 + j]);
                tmem_st32(lane_base + T_SST + (c0 + cc) * 32, w);
            }
#pragma unroll
            for (int c = 0; c < 64; c += 8) {
                uint32_t pk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) pk[j] = pack_bf16x2(srow[c + 2 * j], srow[c + 2 * j + 1]);
                st_shared_v4(sbase + MS_S + swz(r, hc * 64 + c), pk);
            }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        if (!(a.debug_flags & SFA_DEBUG_STALL_GDN_STATE)) mbar_arrive(s_ready);
        pdl_wait();  // B_N comes from the preparation kernel
        bool ok = true;
        int it = 0;
        // O of tile it -> bf16 into its Q buffer, for the TMA warp's store
        auto stage_o = [&]() -> bool {
            const int u = it & 1;
            if (!__all_sync(0xffffffffu, gwait(o_done(u), (it >> 1) & 1, abort, a.status, a.timeout_ns)))
                return false;
            tc_fence_after();
            const uint32_t qb = sbase + MS_Q + (it % NQ) * G_TILE;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = c0 + cc;
                uint32_t v[32];
                tmem_ld32(lane_base + T_O0 + u * 128 + c * 32, v);
                tmem_wait_ld_regs(v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        w[j] = pack_bf16x2(__uint_as_float(v[8 * q + 2 * j]), __uint_as_float(v[8 * q + 2 * j + 1]));
                    st_shared_v4(qb + swz(r, c * 32 + q * 8), w);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(o_staged(it % NQ));
            ++it;
            return true;
        };
        for (int n = 0; n < a.T && ok; ++n) {
            // the frame's O products past its second wait for the TMEM buffers of its first
            // ones, and the frame's MMAs end before the state is rewritten: those first ones
            // are staged before the state
            const int per = tiles_in(n);
            const int early = upd ? (per > 2 ? per - 2 : 0) : per;
            uint32_t pk[32];  // bf16 pairs of the new state row (this half)
            if (upd) {
                // B_N row r (this half), in flight while M_N S is computed: column groups
                // 16 hc .. 16 hc + 15, each load of the warp 512 contiguous bytes
                const float4 *bp = reinterpret_cast<const float4 *>(a.bws) + ((bhi * a.T + n) * 32 + hc * 16) * GD + r;
                float4 bn[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) bn[j] = __ldg(bp + j * GD);
                const float al = a.alpha[bhi * a.T + n];
                if (!(ok = __all_sync(0xffffffffu, gwait(d_done, n & 1, abort, a.status, a.timeout_ns)))) break;
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = c0 + cc;
                    uint32_t dv[32], sv[32];
                    tmem_ld32(lane_base + T_D + c * 32, dv);
                    tmem_ld32(lane_base + T_SST + c * 32, sv);
                    tmem_wait_ld_regs(dv);
                    tmem_wait_ld_regs(sv);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float4 b4 = bn[cc * 8 + j / 4];
                        const float bj = (j & 3) == 0 ? b4.x : (j & 3) == 1 ? b4.y : (j & 3) == 2 ? b4.z : b4.w;
                        sv[j] = __float_as_uint(fmaf(al, __uint_as_float(sv[j]), bj - __uint_as_float(dv[j])));
                    }
                    tmem_st32(lane_base + T_SST + c * 32, sv);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[cc * 16 + j] = pack_bf16x2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]));
                }
            }
            for (int ii = 0; ii < early && ok; ++ii) ok = stage_o();
            if (!ok) break;
            if (upd) {
                // the frame's MMAs still read bf16(S_{n-1})
                if (!(ok = __all_sync(0xffffffffu, gwait(s_free, n & 1, abort, a.status, a.timeout_ns)))) break;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t w[4] = {pk[cc * 16 + 4 * q], pk[cc * 16 + 4 * q + 1], pk[cc * 16 + 4 * q + 2],
                                               pk[cc * 16 + 4 * q + 3]};
                        st_shared_v4(sbase + MS_S + swz(r, (c0 + cc) * 32 + q * 8), w);
                    }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(s_ready);
            }
            for (int ii = early; ii < per && ok; ++ii) ok = stage_o();
        }
        // state out (CTA 0 of the head; all hold the same state)
        if (ok && a.s_out && g == 0) {
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = c0 + cc;
                uint32_t s[32];
                tmem_ld32(lane_base + T_SST + c * 32, s);
                tmem_wait_ld_regs(s);
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 w = make_float4(__uint_as_float(s[j]), __uint_as_float(s[j + 1]), __uint_as_float(s[j + 2]),
                                           __uint_as_float(s[j + 3]));
                    *reinterpret_cast<float4 *>(a.s_out + (bhi * GD + r) * GD + c * 32 + j) = w;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == GW_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    } else if (warp == GW_TMA && *abort) {
        // copies still in flight (issued, never seen landing by the MMA warp) land before
        // the CTA exits
        for (int x = landed[0]; x < q_loaded; ++x) gdrain(q_full(x % NQ), (x / NQ) & 1);
        for (int x = landed[1]; x < m_loaded; ++x) gdrain(m_full(x & 1), (x >> 1) & 1);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 [B][H][T*P][d] as a 5-D map (d, P, T, H, B), box 64 x rows x 1 x 1 x 1, 128-byte
// swizzle: a tile never crosses its frame; rows past the frame read as zero and are not
// written by a store
bool encode_frames(CUtensorMap *m, const void *base, int B, int H, int T, int P, const int64_t *stride,
                   int rows = GBM)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gd[5] = {(cuuint64_t)GD, (cuuint64_t)P, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t gs[4] = {(cuuint64_t)stride[2] * 2, (cuuint64_t)P * stride[2] * 2, (cuuint64_t)stride[1] * 2,
                              (cuuint64_t)stride[0] * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)rows, 1, 1, 1}, es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), gd, gs, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows][d] row-major (M_N) as a 2-D map with a 128-byte-swizzled box of 128 rows x
// 64 columns
bool encode_rows(CUtensorMap *m, void *base, int64_t rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gd[2] = {(cuuint64_t)GD, (cuuint64_t)rows};
    const cuuint64_t gs[1] = {(cuuint64_t)GD * 2};
    const cuuint32_t box[2] = {64, 128}, es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, gd, gs, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gdn_stride_ok(const int64_t *s)
{
    return s[2] >= GD && s[0] >= 0 && s[1] >= 0 && s[0] % 8 == 0 && s[1] % 8 == 0 && s[2] % 8 == 0;
}

// CTAs per (batch, head) in gdn_kernel: as many as fill the SMs once, at most one per tile
int gdn_split(const sfa_gdn_desc *d)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tiles = (d->P + GBM - 1) / GBM;
    const int64_t heads = (int64_t)d->B * d->H;
    return (int)std::max<int64_t>(1, std::min<int64_t>(n_tiles, sms / heads));
}

// workspace: M_N bf16 [B*H*T][d][d], then B_N fp32 [B*H*T][32][d][4] (see GdnArgs::bws)
size_t gdn_m_bytes(const sfa_gdn_desc *d) { return (size_t)d->B * d->H * d->T * GD * GD * 2; }
size_t gdn_ws_bytes(const sfa_gdn_desc *d) { return gdn_m_bytes(d) * 3; }

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_gdn_workspace(const sfa_gdn_desc *d, size_t *bytes)
{
    if (!d || !bytes || d->B < 0 || d->H < 1 || d->T < 1 || d->P < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != GD) return SFA_ERR_UNSUPPORTED;
    *bytes = gdn_ws_bytes(d);
    return SFA_OK;
}

extern "C" sfa_status sfa_gdn_forward(const sfa_gdn_desc *d, const void *q, const void *k, const void *v,
                                      const float *alpha, const float *beta, const float *state_in,
                                      float *state_out, void *o, int32_t update, void *workspace,
                                      size_t workspace_bytes, int32_t *dev_status, sfa_stream_t stream)
{
    if (!d || d->B < 0 || d->H < 1 || d->T < 1 || d->P < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != GD) return SFA_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->P >= ((int64_t)1 << 31) || (int64_t)d->B * d->H * d->T * GD >= ((int64_t)1 << 31))
        return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!q || !k || !v || !o || !alpha || !beta || !state_out) return SFA_ERR_INVALID_ARG;
    const void *ptrs[5] = {q, k, v, o, state_out};
    for (const void *p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) % 16) return SFA_ERR_INVALID_ARG;
    if (state_in && reinterpret_cast<uintptr_t>(state_in) % 16) return SFA_ERR_INVALID_ARG;
    if (!gdn_stride_ok(d->q_stride) || !gdn_stride_ok(d->k_stride) || !gdn_stride_ok(d->v_stride) ||
        !gdn_stride_ok(d->o_stride))
        return SFA_ERR_INVALID_ARG;
    if (update && (!workspace || workspace_bytes < gdn_ws_bytes(d) || reinterpret_cast<uintptr_t>(workspace) % 256))
        return SFA_ERR_INVALID_ARG;
    CUtensorMap tq, to, tm;
    if (!encode_frames(&tq, q, d->B, d->H, d->T, d->P, d->q_stride) ||
        !encode_frames(&to, o, d->B, d->H, d->T, d->P, d->o_stride))
        return SFA_ERR_UNSUPPORTED;
    std::memset(&tm, 0, sizeof(tm));  // read only when the state is updated
    GdnArgs a;
    a.B = d->B;
    a.H = d->H;
    a.T = d->T;
    a.P = d->P;
    a.n_tiles = (d->P + GBM - 1) / GBM;
    a.update = update ? 1 : 0;
    a.G = gdn_split(d);
    a.alpha = alpha;
    a.beta = beta;
    a.s_in = state_in;
    a.s_out = state_out;
    a.bws = nullptr;
    a.status = dev_status;
    a.timeout_ns = (uint64_t)(d->timeout_us ? d->timeout_us : 2000000u) * 1000;
    a.debug_flags = d->debug_flags;
    cudaStream_t s = as_cuda(stream);
    if (update) {
        const int64_t rows = (int64_t)d->B * d->H * d->T * GD;
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        CUtensorMap tk, tv;
        if (!encode_frames(&tk, k, d->B, d->H, d->T, d->P, d->k_stride, PBM) ||
            !encode_frames(&tv, v, d->B, d->H, d->T, d->P, d->v_stride, PBM) || !encode_rows(&tm, ws, rows))
            return SFA_ERR_UNSUPPORTED;
        a.bws = reinterpret_cast<const float *>(ws + gdn_m_bytes(d));
        if (cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PR_SMEM) !=
            cudaSuccess)
            return SFA_ERR_CUDA;
        gdn_prep_kernel<<<(unsigned)(d->B * d->H * d->T), GTHREADS, PR_SMEM, s>>>(tk, tv, tm, a);
        if (cudaGetLastError() != cudaSuccess) return SFA_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MS_SMEM) != cudaSuccess)
        return SFA_ERR_CUDA;
    // after the preparation kernel: a programmatic dependent launch, so that the recurrence
    // kernel's set-up (barriers, tensor memory, its first Q tiles, the input state) overlaps
    // the preparation's last CTAs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(d->B * d->H * a.G));
    cfg.blockDim = dim3(GTHREADS_REC);
    cfg.dynamicSmemBytes = MS_SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = update ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, gdn_kernel, tq, to, tm, a) != cudaSuccess) return SFA_ERR_CUDA;
    return launch_status();
}
