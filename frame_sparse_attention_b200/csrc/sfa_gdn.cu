// ARL2 inter-frame branch: gated delta rule with frame-level state access, sm_100a.
//
// "Resumen Técnico: Asistir Localmente, Recordar Linealmente (ARL2)", §2.1 (Rama
// Inter-Cuadro): a fixed-size state S [d x d] per (batch, head) replaces the KV cache;
// frame N reads it as O_N = Q'_N S_{N-1} and then updates it as
//   S_N = alpha_N S_{N-1} + K'_N^T diag(beta_N) (V'_N - K'_N S_{N-1});
// §2.2: every token of a frame reads the same pre-update state (frame-level access), and
// intermediate denoising steps read without writing (update = 0).
//
// Because the state changes once per frame, a frame is three dense contractions on the
// tensor cores, tile by tile (128 tokens):
//   O  = Q_i S           (M = 128 tokens, N = d, K = d; S as the B operand, bf16)
//   KS = K_i S           (same)
//   S_acc += K_i^T U_i   (M = d, N = d, K = 128 tokens), U_i = diag(beta) (V_i - KS)
// G CTAs per (batch, head) run the frames in order (the recurrence is sequential); CTA g
// takes tiles g, g + G, ... of every frame, and its tiles form one sequence over the frames
// through two shared-memory slots, so the copies of the next tile are in flight while the
// current one computes.  With G > 1 each CTA adds its partial S_acc into one fp32 sum per
// head with a TMA reduce-add (performed in L2), the G CTAs of a head meet at a counter in
// global memory (one cooperative launch, so all CTAs are resident; the wait is bounded),
// and each copies the sum back with one TMA load.  The sums rotate over three buffers by
// frame: buffer n mod 3 is summed into in frame n, and CTA 0 zeroes buffer (n + 2) mod 3
// after the meeting of frame n, when every CTA has finished reading it (frame n - 1) and
// none can add into it yet (frame n + 2 comes after the next meeting); one meeting per
// frame is enough.  Per tile the MMAs run KS first, then O, then (once U is in shared
// memory) S_acc.  Warps 0-7 (two threads per TMEM lane, 64 columns each) form U over V,
// stage O in the tile's Q buffer and update the fp32 state; warp 8 issues the TMA copies,
// the MMAs and the TMA stores of O.
// Read-only steps (update = 0) leave the state alone, so their frames are independent.
// Tensor memory: O, KS, S_acc and the fp32 state, 128 columns each.  Every wait is
// bounded; a wait that runs out stores SFA_ERR_TIMEOUT and the CTA drains and exits.
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
constexpr int GEPI = 256;        // warps 0-7: epilogue (two threads per TMEM lane)
constexpr int GW_MMA = 8;        // warp 8: TMA copies and MMAs
constexpr int GTHREADS = GEPI + 32;
constexpr int G_BOX = 128 * 128; // one 128-row x 64-column bf16 box (128-byte swizzle)
constexpr int G_TILE = 2 * G_BOX;
constexpr int F_BOX = 128 * 128; // one 128-row x 32-column fp32 box (128-byte swizzle)
// shared memory: the bf16 state (B operand of O and KS), then two slots of Q, K, V for
// consecutive tiles (U is written over V); at a frame end the Q and K of the slot of the
// frame's last tile stage the partial S_acc and then the head's sum (64 KB fp32)
constexpr int G_S = 0, G_SLOT0 = G_TILE, G_SLOT_BYTES = 3 * G_TILE;
constexpr int SL_Q = 0, SL_K = G_TILE, SL_V = 2 * G_TILE;
constexpr int G_BAR = G_SLOT0 + 2 * G_SLOT_BYTES;
constexpr int G_SMEM = G_BAR + 128 + 1024;
constexpr uint32_t T_O = 0, T_KS = 128, T_SACC = 256, T_SST = 384;  // tensor-memory columns

struct GdnArgs {
    int32_t B, H, T, P, n_tiles, update;
    int32_t G;           // CTAs per (batch, head)
    float *part;         // [3][B*H][d][d] sums of the partial S_acc (G > 1 with update), zero at launch
    uint32_t *count;     // [B*H] arrivals (G > 1 with update), zero at launch
    const float *alpha;  // [B][H][T]
    const float *beta;   // [B][H][T*P]
    const float *s_in;   // [B][H][d][d] or null (zeros)
    float *s_out;        // [B][H][d][d]
    int32_t *status;
    uint64_t timeout_ns;
};

struct GBars {
    uint32_t base;
    __device__ uint32_t full(uint32_t s) const { return base + 8 * s; }  // Q, K, V of slot s landed
    __device__ uint32_t ks() const { return base + 16; }       // KS of a tile in TMEM
    __device__ uint32_t o() const { return base + 24; }        // O of a tile in TMEM
    __device__ uint32_t u_full() const { return base + 32; }   // U in smem, KS read (all epilogue threads)
    __device__ uint32_t o_free() const { return base + 40; }   // O read out of TMEM into the Q buffer (all)
    __device__ uint32_t sacc() const { return base + 48; }     // S_acc MMA of a tile done
    __device__ uint32_t s_ready() const { return base + 56; }  // state for the next frame (all)
    __device__ uint32_t sum() const { return base + 64; }      // the head's summed S_acc landed
    __device__ uint32_t drain() const { return base + 72; }
    __device__ uint32_t staged() const { return base + 80; }   // partial S_acc staged (all)
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

// byte offset of fp32 columns 32 c + 4 j .. + 3 of row r in four swizzled 32-column boxes
// (the layout a 128-byte-swizzle TMA copy of a 32 x 128 fp32 box uses)
__device__ __forceinline__ uint32_t fswz(int r, int c, int j)
{
    return (uint32_t)(c * F_BOX + r * 128 + ((j ^ (r & 7)) << 4));
}

__device__ __forceinline__ float bf16f(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

__global__ void __launch_bounds__(GTHREADS, 1)
    gdn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const __grid_constant__ CUtensorMap tm_part, const __grid_constant__ GdnArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const GBars bar{sbase + G_BAR};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + G_BAR + 112);
    volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(smem + G_BAR + 116);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x / a.G, g = blockIdx.x % a.G, b = bh / a.H, h = bh % a.H;
    const bool upd = a.update != 0, spread = upd && a.G > 1;  // spread: partial updates summed over the head's CTAs
    const int per = (a.n_tiles - g + a.G - 1) / a.G;          // tiles of a frame this CTA takes: g, g + G, ...

    if (threadIdx.x == 0) {
        const uint32_t single[7] = {bar.full(0), bar.full(1), bar.ks(), bar.o(), bar.sacc(), bar.sum(), bar.drain()};
        for (uint32_t x : single) mbar_init(x, 1);
        const uint32_t all[4] = {bar.u_full(), bar.o_free(), bar.s_ready(), bar.staged()};
        for (uint32_t x : all) mbar_init(x, GEPI);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == GW_MMA) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_o);
            if (spread) tma_prefetch_desc(&tm_part);
        }
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == GW_MMA) {
        // ---------------------------------------------------------------- TMA + MMA
        // The CTA's tiles form one sequence over the frames (tile t: frame t / per); tile t
        // uses slot t & 1, and its copies are issued while tile t - 1 is in flight.
        const uint64_t ds = sdesc_sw128(sbase + G_S, G_BOX, 1024);    // S: [d_k rows][d_v], MN-major B
        constexpr uint32_t id_qs = idesc_bf16_f32(GBM, GD, true);
        constexpr uint32_t id_kt = idesc_bf16_f32(GD, GD, true) | (1u << 15);  // A MN-major
        const uint32_t total = (uint32_t)per * (uint32_t)a.T;
        uint32_t n_loaded = 0, n_landed = 0;  // tiles whose copies were issued / seen landed here
        bool ok = true, issued = false;
        auto load = [&](uint32_t t) {
            const uint32_t dst = sbase + G_SLOT0 + (t & 1) * G_SLOT_BYTES;
            const int n = (int)(t / per), i = g + (int)(t % per) * a.G;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar.full(t & 1), 3 * G_TILE);
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    tma_load_5d(dst + SL_K + kb * G_BOX, &tm_k, bar.full(t & 1), kb * 64, i * GBM, n, h, b);
                    tma_load_5d(dst + SL_Q + kb * G_BOX, &tm_q, bar.full(t & 1), kb * 64, i * GBM, n, h, b);
                    tma_load_5d(dst + SL_V + kb * G_BOX, &tm_v, bar.full(t & 1), kb * 64, i * GBM, n, h, b);
                }
            }
            __syncwarp();
            n_loaded = t + 1;
        };
        // O of tile t (staged by the epilogue in its Q buffer) -> global; lane 0 owns the
        // bulk groups
        auto store_o = [&](uint32_t t) {
            const uint32_t src = sbase + G_SLOT0 + (t & 1) * G_SLOT_BYTES + SL_Q;
            const int n = (int)(t / per), i = g + (int)(t % per) * a.G;
            if (lane == 0) {
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) tma_store_5d(&tm_o, src + kb * G_BOX, kb * 64, i * GBM, n, h, b);
                tma_store_commit();
            }
            __syncwarp();
        };
        if (total > 0) load(0);
        for (uint32_t it = 0; it < total && ok; ++it) {
            const uint32_t n = it / per, ii = it % per, slot = it & 1;
            // a frame starts from the state of the previous one (read-only steps: the input state)
            if (ii == 0 && (upd || n == 0) &&
                !(ok = __all_sync(0xffffffffu, gwait(bar.s_ready(), n & 1, abort, a.status, a.timeout_ns))))
                break;
            if (!(ok = __all_sync(0xffffffffu, gwait(bar.full(slot), (it >> 1) & 1, abort, a.status, a.timeout_ns))))
                break;
            n_landed = it + 1;
            tc_fence_after();
            const uint32_t sl = sbase + G_SLOT0 + slot * G_SLOT_BYTES;
            const uint64_t dq = sdesc_sw128(sl + SL_Q, 16, 1024);   // Q tile, K-major A
            const uint64_t dk = sdesc_sw128(sl + SL_K, 16, 1024);   // K tile, K-major A
            if (upd) {  // KS first: U waits for it (KS of the previous tile was read before its U)
                if (elect_one()) {
#pragma unroll
                    for (uint32_t kk = 0; kk < GD / 16; ++kk) {
                        const uint32_t ka = (kk >> 2) * G_BOX + (kk & 3) * 32;
                        mma_ss(tmem + T_KS, dk + (ka >> 4), ds + ((kk * 2048) >> 4), id_qs, kk > 0);
                    }
                    tc_commit(bar.ks());
                }
                __syncwarp();
                issued = true;
            }
            // O of the previous tile read out of TMEM and staged: its store goes out (a frame's
            // last tile went out already, during the frame end)
            if (it > 0 && ii != 0) {
                if (!(ok = __all_sync(0xffffffffu, gwait(bar.o_free(), (it - 1) & 1, abort, a.status, a.timeout_ns))))
                    break;
                store_o(it - 1);
            }
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (uint32_t kk = 0; kk < GD / 16; ++kk) {
                    const uint32_t ka = (kk >> 2) * G_BOX + (kk & 3) * 32;
                    mma_ss(tmem + T_O, dq + (ka >> 4), ds + ((kk * 2048) >> 4), id_qs, kk > 0);
                }
                tc_commit(bar.o());
            }
            __syncwarp();
            issued = true;
            if (it + 1 < total) {
                // the other slot last held tile it - 1: its S_acc MMA is done, its O tile's
                // store has read the Q buffer, and (at a frame start) the staged sums of the
                // frame before were read by the time the state was ready
                if (upd && it > 0 &&
                    !(ok = __all_sync(0xffffffffu, gwait(bar.sacc(), (it - 1) & 1, abort, a.status, a.timeout_ns))))
                    break;
                if (lane == 0) tma_store_wait_read_all();
                __syncwarp();
                load(it + 1);
            }
            if (upd) {
                if (!(ok = __all_sync(0xffffffffu, gwait(bar.u_full(), it & 1, abort, a.status, a.timeout_ns))))
                    break;
                tc_fence_after();
                const uint64_t dkt = sdesc_sw128(sl + SL_K, G_BOX, 1024);  // K tile read as K^T: MN-major A
                const uint64_t du = sdesc_sw128(sl + SL_V, G_BOX, 1024);   // U tile, MN-major B
                if (elect_one()) {
                    // S_acc += K^T U over the tile's 128 tokens, 16 per step
#pragma unroll
                    for (uint32_t kk = 0; kk < GBM / 16; ++kk)
                        mma_ss(tmem + T_SACC, dkt + ((kk * 2048) >> 4), du + ((kk * 2048) >> 4), id_kt,
                               (ii > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar.sacc());
                }
                __syncwarp();
            }
            if (ii + 1 == (uint32_t)per) {  // the frame's last tile: its O goes out now
                if (!(ok = __all_sync(0xffffffffu, gwait(bar.o_free(), it & 1, abort, a.status, a.timeout_ns))))
                    break;
                store_o(it);
            }
        }
        if (lane == 0) bulk_commit_and_wait_all();  // every O store complete
        __syncwarp();
        if (__any_sync(0xffffffffu, *abort != 0)) {
            if (issued) {  // tensor cores idle before TMEM is freed
                if (elect_one()) tc_commit(bar.drain());
                __syncwarp();
                gdrain(bar.drain(), 0);
            }
            // copies still in flight land before the CTA exits
            for (uint32_t t = n_landed; t < n_loaded; ++t) gdrain(bar.full(t & 1), (t >> 1) & 1);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue, row r, half hc
        // warps w and w + 4 share TMEM lanes 32 (w mod 4) .. + 31 (tile rows, state rows) and
        // take 64 columns each
        const int e = threadIdx.x, qd = warp & 3, hc = warp >> 2;
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
                st_shared_v4(sbase + G_S + swz(r, hc * 64 + c), pk);
            }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar.s_ready());
        bool ok = true;
        int sum_n = -1;  // thread 0: the frame whose sum is being copied in, or -1
        uint32_t it = 0;
        // beta of this thread's row in the CTA's tile t (0 past the frame), loaded a tile ahead
        auto beta_of = [&](uint32_t t) {
            const int n = (int)(t / per), row = (g + (int)(t % per) * a.G) * GBM + r;
            return (upd && n < a.T && row < a.P) ? a.beta[(bhi * a.T + n) * a.P + row] : 0.f;
        };
        float bt_next = beta_of(0);
        for (int n = 0; n < a.T && ok; ++n) {
            const float al = upd ? a.alpha[bhi * a.T + n] : 0.f;
            for (int ii = 0; ii < per; ++ii, ++it) {
                const uint32_t sl = G_SLOT0 + (it & 1) * G_SLOT_BYTES;
                const float bt = bt_next;
                bt_next = beta_of(it + 1);
                if (upd) {
                    ok = __all_sync(0xffffffffu, gwait(bar.ks(), it & 1, abort, a.status, a.timeout_ns)) &&
                         __all_sync(0xffffffffu, gwait(bar.full(it & 1), (it >> 1) & 1, abort, a.status, a.timeout_ns));
                    if (!ok) break;
                    tc_fence_after();
                    // U row = beta_row (V row - KS row) -> bf16, written over the V row
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = c0 + cc;
                        uint32_t ks[32];
                        tmem_ld32(lane_base + T_KS + c * 32, ks);
                        tmem_wait_ld_regs(ks);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t off = sl + SL_V + swz(r, c * 32 + q * 8);
                            const uint4 vv = *reinterpret_cast<const uint4 *>(smem + off);
                            const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                            uint32_t pk[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float v0 = bf16f((uint16_t)(vw[j] & 0xffffu)), v1 = bf16f((uint16_t)(vw[j] >> 16));
                                pk[j] = pack_bf16x2(bt * (v0 - __uint_as_float(ks[8 * q + 2 * j])),
                                                    bt * (v1 - __uint_as_float(ks[8 * q + 2 * j + 1])));
                            }
                            st_shared_v4(sbase + off, pk);
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(bar.u_full());
                }
                if (!(ok = __all_sync(0xffffffffu, gwait(bar.o(), it & 1, abort, a.status, a.timeout_ns)))) break;
                tc_fence_after();
                // O row -> bf16 into the Q buffer (read by the finished O MMA), in the layout of
                // the output's tensor map; the MMA warp's TMA store writes the tile
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = c0 + cc;
                    uint32_t v[32];
                    tmem_ld32(lane_base + T_O + c * 32, v);
                    tmem_wait_ld_regs(v);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            w[j] = pack_bf16x2(__uint_as_float(v[8 * q + 2 * j]), __uint_as_float(v[8 * q + 2 * j + 1]));
                        st_shared_v4(sbase + sl + SL_Q + swz(r, c * 32 + q * 8), w);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar.o_free());
            }
            if (!ok || !upd) continue;
            // frame end: S <- alpha S + S_acc (summed over the head's CTAs), fp32 in TMEM,
            // bf16 copy for the next frame
            ok = __all_sync(0xffffffffu, gwait(bar.sacc(), (it - 1) & 1, abort, a.status, a.timeout_ns));
            if (!ok) break;
            tc_fence_after();
            const uint32_t stage = G_SLOT0 + ((it - 1) & 1) * G_SLOT_BYTES + SL_K;  // K and U of the last tile
            if (spread) {
                // this CTA's partial, swizzled like the fp32 boxes of the sum's tensor map
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = c0 + cc;
                    uint32_t acc[32];
                    tmem_ld32(lane_base + T_SACC + c * 32, acc);
                    tmem_wait_ld_regs(acc);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t w[4] = {acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]};
                        st_shared_v4(sbase + stage + fswz(r, c, j), w);
                    }
                }
                fence_proxy_async_smem();
                // (the arrival also orders this thread's zeroing of the frame before ahead of
                // thread 0's release of the CTA's next arrival at the counter)
                mbar_arrive(bar.staged());
                if (e == 0 && gwait(bar.staged(), n & 1, abort, a.status, a.timeout_ns)) {
                    // add it into the head's sum in L2, meet the head's other CTAs, fetch the sum
                    const int y = ((n % 3) * a.B * a.H + bh) * GD;
#pragma unroll
                    for (int c = 0; c < GD / 32; ++c) tma_reduce_add_2d(&tm_part, sbase + stage + c * F_BOX, c * 32, y);
                    bulk_commit_and_wait_all();
                    red_release_add(a.count + bh, 1u);
                    const uint32_t want = (uint32_t)a.G * (uint32_t)(n + 1);
                    const uint64_t t0 = gns();
                    for (uint32_t spins = 0; ld_acquire(a.count + bh) < want; ++spins) {
                        if (*abort) break;
                        if ((spins & 63) == 63 && gns() - t0 > a.timeout_ns) {
                            *abort = 1;
                            if (a.status) atomicCAS(a.status, 0, SFA_ERR_TIMEOUT);
                            break;
                        }
                    }
                    fence_proxy_async_global();
                    if (!*abort) {
                        mbar_arrive_expect_tx(bar.sum(), 4 * F_BOX);
#pragma unroll
                        for (int c = 0; c < GD / 32; ++c)
                            tma_load_2d(sbase + stage + c * F_BOX, &tm_part, bar.sum(), c * 32, y);
                        sum_n = n;
                    }
                }
                // (a warp that left on an abort never arrives: every wait here is bounded)
                if (!(ok = __all_sync(0xffffffffu, gwait(bar.sum(), n & 1, abort, a.status, a.timeout_ns)))) break;
                sum_n = -1;
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int c = c0 + cc;
                uint32_t s[32], acc[32];
                tmem_ld32(lane_base + T_SST + c * 32, s);
                tmem_wait_ld_regs(s);
                if (spread) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 v4 = *reinterpret_cast<const uint4 *>(smem + stage + fswz(r, c, j));
                        acc[4 * j] = v4.x;
                        acc[4 * j + 1] = v4.y;
                        acc[4 * j + 2] = v4.z;
                        acc[4 * j + 3] = v4.w;
                    }
                } else {
                    tmem_ld32(lane_base + T_SACC + c * 32, acc);
                    tmem_wait_ld_regs(acc);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    s[j] = __float_as_uint(fmaf(al, __uint_as_float(s[j]), __uint_as_float(acc[j])));
                tmem_st32(lane_base + T_SST + c * 32, s);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t pk[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        pk[j] = pack_bf16x2(__uint_as_float(s[8 * q + 2 * j]), __uint_as_float(s[8 * q + 2 * j + 1]));
                    st_shared_v4(sbase + G_S + swz(r, c * 32 + q * 8), pk);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar.s_ready());
            if (spread) {
                // buffer (n + 2) mod 3 was read by every CTA in frame n - 1 and is next summed
                // into in frame n + 2, after every CTA's arrival of frame n + 1: CTA g zeroes
                // its share of it now (released by thread 0's next arrival)
                float4 *z = reinterpret_cast<float4 *>(a.part + ((int64_t)((n + 2) % 3) * a.B * a.H + bh) * GD * GD);
                const int z0 = g * (GD * GD / 4) / a.G, z1 = (g + 1) * (GD * GD / 4) / a.G;
                for (int j = z0 + e; j < z1; j += GEPI) __stcg(z + j, make_float4(0.f, 0.f, 0.f, 0.f));
            }
        }
        if (sum_n >= 0) gdrain(bar.sum(), (uint32_t)sum_n & 1);
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

// bf16 [B][H][T*P][d] as a 5-D map (d, P, T, H, B), box 64 x 128 x 1 x 1 x 1, 128-byte
// swizzle: a tile never crosses its frame; rows past the frame read as zero and are not
// written by a store
bool encode_frames(CUtensorMap *m, const void *base, int B, int H, int T, int P, const int64_t *stride)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gd[5] = {(cuuint64_t)GD, (cuuint64_t)P, (cuuint64_t)T, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t gs[4] = {(cuuint64_t)stride[2] * 2, (cuuint64_t)P * stride[2] * 2, (cuuint64_t)stride[1] * 2,
                              (cuuint64_t)stride[0] * 2};
    const cuuint32_t box[5] = {64, (cuuint32_t)GBM, 1, 1, 1}, es[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), gd, gs, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the fp32 sums [3 * B * H * d rows][d] as a 2-D map, box 32 columns x 128 rows, 128-byte
// swizzle: four boxes hold one head's d x d sum
bool encode_part(CUtensorMap *m, float *part, int64_t rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gd[2] = {(cuuint64_t)GD, (cuuint64_t)rows};
    const cuuint64_t gs[1] = {(cuuint64_t)GD * 4};
    const cuuint32_t box[2] = {32, 128}, es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, part, gd, gs, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gdn_stride_ok(const int64_t *s)
{
    return s[2] >= GD && s[0] >= 0 && s[1] >= 0 && s[0] % 8 == 0 && s[1] % 8 == 0 && s[2] % 8 == 0;
}

// CTAs per (batch, head): about two tiles of a frame each, all resident at once (one CTA
// per SM: the kernel's shared memory allows no second one)
int gdn_split(const sfa_gdn_desc *d)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tiles = (d->P + GBM - 1) / GBM;
    const int64_t heads = (int64_t)d->B * d->H;
    int G = (n_tiles + 1) / 2;
    if (heads * G > sms) G = (int)std::max<int64_t>(1, sms / heads);
    return std::max(G, 1);
}

size_t gdn_part_bytes(const sfa_gdn_desc *d, int)
{
    return ((size_t)3 * d->B * d->H * GD * GD * 4 + 255) / 256 * 256;
}

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_gdn_workspace(const sfa_gdn_desc *d, size_t *bytes)
{
    if (!d || !bytes || d->B < 0 || d->H < 1 || d->T < 1 || d->P < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != GD) return SFA_ERR_UNSUPPORTED;
    const int G = gdn_split(d);
    *bytes = G > 1 ? gdn_part_bytes(d, G) + ((size_t)d->B * d->H * 4 + 255) / 256 * 256 : 0;
    return SFA_OK;
}

extern "C" sfa_status sfa_gdn_forward(const sfa_gdn_desc *d, const void *q, const void *k, const void *v,
                                      const float *alpha, const float *beta, const float *state_in,
                                      float *state_out, void *o, int32_t update, void *workspace,
                                      size_t workspace_bytes, int32_t *dev_status, sfa_stream_t stream)
{
    if (!d || d->B < 0 || d->H < 1 || d->T < 1 || d->P < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != GD) return SFA_ERR_UNSUPPORTED;
    if ((int64_t)d->T * d->P >= ((int64_t)1 << 31) || (int64_t)d->B * d->H >= ((int64_t)1 << 31))
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
    CUtensorMap tq, tk, tv, to;
    if (!encode_frames(&tq, q, d->B, d->H, d->T, d->P, d->q_stride) ||
        !encode_frames(&tk, k, d->B, d->H, d->T, d->P, d->k_stride) ||
        !encode_frames(&tv, v, d->B, d->H, d->T, d->P, d->v_stride) ||
        !encode_frames(&to, o, d->B, d->H, d->T, d->P, d->o_stride))
        return SFA_ERR_UNSUPPORTED;
    GdnArgs a;
    a.B = d->B;
    a.H = d->H;
    a.T = d->T;
    a.P = d->P;
    a.n_tiles = (d->P + GBM - 1) / GBM;
    a.update = update ? 1 : 0;
    a.alpha = alpha;
    a.beta = beta;
    a.s_in = state_in;
    a.s_out = state_out;
    a.status = dev_status;
    a.timeout_ns = (uint64_t)(d->timeout_us ? d->timeout_us : 2000000u) * 1000;
    // read-only steps: the frames are independent, so the tiles spread over several CTAs per
    // head without meeting; updating steps spread them only with the workspace, through which
    // the CTAs exchange their partial updates, and one CTA per head otherwise
    const int G = (workspace || !update) ? gdn_split(d) : 1;
    a.G = G;
    a.part = nullptr;
    a.count = nullptr;
    CUtensorMap tp;
    std::memset(&tp, 0, sizeof(tp));  // read only by CTAs that exchange partial updates
    cudaStream_t s = as_cuda(stream);
    if (cudaFuncSetAttribute(gdn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM) != cudaSuccess)
        return SFA_ERR_CUDA;
    if (G > 1 && update) {
        const size_t pb = gdn_part_bytes(d, G), need = pb + ((size_t)d->B * d->H * 4 + 255) / 256 * 256;
        if (workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256) return SFA_ERR_INVALID_ARG;
        a.part = static_cast<float *>(workspace);
        a.count = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + pb);
        if (!encode_part(&tp, a.part, (int64_t)3 * d->B * d->H * GD)) return SFA_ERR_UNSUPPORTED;
        if (cudaMemsetAsync(workspace, 0, need, s) != cudaSuccess) return SFA_ERR_CUDA;  // sums and counters
        // the G CTAs of a head wait for one another: one cooperative launch keeps them all resident
        void *args[] = {&tq, &tk, &tv, &to, &tp, &a};
        const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(gdn_kernel),
                                                          dim3((unsigned)(d->B * d->H * G)), dim3(GTHREADS), args,
                                                          G_SMEM, s);
        return e == cudaSuccess ? launch_status() : SFA_ERR_CUDA;
    }
    gdn_kernel<<<(unsigned)(d->B * d->H * G), GTHREADS, G_SMEM, s>>>(tq, tk, tv, to, tp, a);
    return launch_status();
}
