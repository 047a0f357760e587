// Frame-sparse softmax attention forward for sm_100a (B200).
//
// What it computes ("LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de
// Video Largo", §2 Mecanismo Central and §Complejidad): every query frame t attends only
// to the key/value tokens of the frames in A(h, t), so a query costs O(|A| P d) instead
// of O(T P d).  Per row it also emits the log-sum-exp of its scaled scores, the state
// that "ISPA" (§2.1, Atención Descomponible) uses to merge partial attentions.
//
// How, on one SM per work unit (b, h, t, pair of 128-row query tiles A and B):
//   * the frame list of (h, t) is walked as runs of consecutive frames; each run is one
//     contiguous token interval, cut into 128-key tiles, so unattended frames are never
//     loaded and only the last tile of a run is partial;
//   * warp 8 loads Q of both tiles once and streams K tiles through a 2-slot ring, warp
//     10 streams V tiles (1 slot at d = 128, 2 at d = 64), all with TMA, 128-byte
//     swizzled; a K slot frees once S of both tiles has read it, a V slot once P V of
//     both has;
//   * warp 9 (one elected lane) issues tcgen05.mma for both tiles in the order
//     S_A(0) S_B(0) | P V_A(j) S_A(j+1) P V_B(j) S_B(j+1) ..., S into TMEM (one buffer per
//     tile), O += P V with P read from shared memory (both operands in shared memory: the
//     tensor-memory-A form of this MMA runs at ~0.6x the rate on sm_100); a partial last
//     tile uses an MMA N (for S) and K (for P V) rounded up to 16 only.  While the
//     softmax of one tile runs, the tensor cores work on the other.  A CTA with a single
//     query tile (the last tile of a frame with an odd tile count) uses the idle tile's S
//     and P buffers as second buffers and runs S two key tiles ahead instead;
//   * warps 0-3 (tile A) and 4-7 (tile B), one thread per query row = TMEM lane, run the
//     online softmax in fp32 (exp2 with the scale folded into one FMA; O is rescaled only
//     when a row's running max grows by more than 2^8, otherwise the stale max is kept),
//     write P as bf16 into a 128-byte-swizzled shared-memory tile, and finally normalise
//     O, stage it in shared memory and TMA-store it, clipped to the frame, plus the fp32
//     LSE.
// Every mbarrier wait is bounded; a wait that runs out records SFA_ERR_TIMEOUT, the CTA
// drains its in-flight copies and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "sfa.h"
#include "sfa_internal.h"
#include "sfa_ptx.cuh"


namespace sfa {
namespace {

constexpr int BM = 128;                 // query rows per tile = MMA M = TMEM lanes
constexpr int BN = 128;                 // keys per K/V tile (largest MMA N used)
constexpr int KEY_BLOCK = 128;          // tokens per key block of a key-block list
// warps 0-3 softmax of query tile A, 4-7 softmax of query tile B, 8 Q+K loader,
// 9 MMA issuer, 10 V loader
constexpr int NUM_THREADS = 352;
constexpr int K_LOAD_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int V_LOAD_WARP = 10;
constexpr float RESCALE_LIMIT = 256.0f;  // keep a stale row max while the tile's row sum against it stays <= 2^8
constexpr uint32_t DEFAULT_TIMEOUT_US = 2000000;  // 2 s; a healthy wait lasts microseconds
constexpr uint32_t DRAIN_TIMEOUT_US = 2000000;
constexpr uint32_t MAX_SPINS = 1u << 30;           // backstop should the timer not advance

// tensor-memory columns (512 allocated): S of tile A / B, O of tile A / B (fp32)
constexpr uint32_t TM_COLS = 512;
__host__ __device__ constexpr uint32_t tcol_s(int x) { return (uint32_t)x * 128; }
__host__ __device__ constexpr uint32_t tcol_o(int x) { return 256 + (uint32_t)x * 128; }

template <int D>
struct Cfg {
    static constexpr int KBOX = D / 64;                 // 128-byte swizzle boxes per row
    static constexpr int BOX_BYTES = 128 * 128;         // 128 rows x 64 bf16
    static constexpr int TILE_BYTES = BM * D * 2;       // one Q / K / V / O tile
    // K and V rings: a K slot frees once S of both query tiles is computed from it, a V
    // slot once P V of both is (d = 128 leaves room for one V slot only)
    static constexpr int NSK = 2;
    static constexpr int NSV = D == 128 ? 1 : 2;
    static constexpr int P_BYTES = BM * BN * 2;          // one bf16 probability tile
    static constexpr int SMEM_Q = 0;                      // Q tiles A and B
    static constexpr int SMEM_P = 2 * TILE_BYTES;         // P tiles A and B
    static constexpr int SMEM_K = SMEM_P + 2 * P_BYTES;
    static constexpr int SMEM_V = SMEM_K + NSK * TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_V + NSV * TILE_BYTES;
    static constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;  // + barriers, + alignment slack
    static_assert(2 * NSK + 2 * NSV + 10 <= 20, "mbarriers must fit in 160 bytes");
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// mbarrier slots (8 bytes each) at SMEM_BAR
template <int D>
struct Bars {
    uint32_t base;
    __device__ uint32_t k_full(int s) const { return base + 8 * s; }
    __device__ uint32_t k_free(int s) const { return base + 8 * (Cfg<D>::NSK + s); }
    __device__ uint32_t v_full(int s) const { return base + 8 * (2 * Cfg<D>::NSK + s); }
    __device__ uint32_t v_free(int s) const { return base + 8 * (2 * Cfg<D>::NSK + Cfg<D>::NSV + s); }
    __device__ uint32_t q_full() const { return base + 8 * (2 * Cfg<D>::NSK + 2 * Cfg<D>::NSV); }
    __device__ uint32_t s_full(int x) const { return q_full() + 8 + 8 * x; }   // S of query tile x in TMEM
    __device__ uint32_t p_full(int x) const { return q_full() + 24 + 8 * x; }  // P of query tile x in smem
    __device__ uint32_t o_final() const { return q_full() + 40; }              // after the last P V
    __device__ uint32_t drain() const { return q_full() + 48; }
    __device__ uint32_t pv_done() const { return q_full() + 56; }  // one-tile CTAs: a P V complete
    __device__ uint32_t pv_x(int x) const { return q_full() + 64 + 8 * x; }  // P V of query tile x complete
    static constexpr int COUNT = 2 * Cfg<D>::NSK + 2 * Cfg<D>::NSV + 10;
};

struct FwdArgs {
    int32_t B, H, Tq, T_kv, P, Amax;
    int32_t n_qtiles;
    float scale_log2;  // softmax scale * log2(e)
    const int32_t *frames;
    const int32_t *counts;
    const int32_t *slots;  // [H][T_kv] physical frame slot of each logical frame, or null
    int32_t n_slots;       // frames held by the K/V buffers (T_kv without a slot table)
    int32_t nblk;          // > 0: the lists hold key blocks of KEY_BLOCK tokens (nblk per frame),
                           // one list per (b, h, t, query block of 2 tiles); 0: frame lists per (h, t)
    const int32_t *frames2;  // second list set (two-branch launch: grid y = 2 x splits), or null
    const int32_t *counts2;
    int32_t n_lists;         // 1, or 2 with frames2 / counts2
    const int2 *items;       // scheduled launch: one work item per CTA (see schedule_kernel), or null
    int32_t k_first;         // scheduled launch: key-tile ranges of list set 0 (its partial slices)
    float *lse;
    int32_t *status;
    uint64_t timeout_ns;
    uint32_t debug_flags;
};

// ----------------------------------------------------------------- pipeline control
struct Ctl {
    volatile int32_t *abort;
    int32_t *status;
    uint64_t timeout_ns;
};

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report(int32_t *status, int32_t code)
{
    if (status) atomicCAS(status, 0, code);
}

// bounded wait for the phase of `bar` with parity `parity`; false on timeout or abort
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Ctl &c)
{
    const uint64_t t0 = global_ns();
    for (uint32_t spins = 1;; ++spins) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*c.abort) return false;
        if ((spins & 63) == 0 && (global_ns() - t0 > c.timeout_ns || spins >= MAX_SPINS)) {
            *c.abort = 1;
            report(c.status, SFA_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl &c)
{
    return mbar_try_wait(bar, parity) || wait_slow(bar, parity, c);
}

// wait used only while draining after an abort: ignores the abort flag
__device__ __noinline__ void wait_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = global_ns();
    for (uint32_t spins = 1; spins < MAX_SPINS; ++spins) {
        if (mbar_try_wait(bar, parity)) return;
        if ((spins & 63) == 0 && global_ns() - t0 > (uint64_t)DRAIN_TIMEOUT_US * 1000) return;
    }
}

// ----------------------------------------------------------------- attended key tiles
// Physical frame slot of a logical key/value frame: a per-head slot table (paged caches)
// or the identity.
__device__ __forceinline__ int slot_of(const int32_t *srow, int f) { return srow ? __ldg(srow + f) : f; }

// Token interval [lo, hi) of list entry x: frame x (through the slot table) or, with
// key-block lists (nblk > 0), block x % nblk of frame x / nblk.
__device__ __forceinline__ void entry_range(int x, int P, int nblk, const int32_t *srow, int &lo, int &hi)
{
    if (nblk) {
        const int f = x / nblk, b = x - f * nblk;
        lo = f * P + b * KEY_BLOCK;
        hi = f * P + min(b * KEY_BLOCK + KEY_BLOCK, P);
    } else {
        lo = slot_of(srow, x) * P;
        hi = lo + P;
    }
}

// Number of K/V tiles for a list, or -1 if the list is not strictly increasing inside
// [0, n_entries) or a frame's slot lies outside [0, n_slots).  A run is a stretch of
// entries whose token intervals follow one another, i.e. one contiguous token interval.
__device__ int count_tiles(const int32_t *fl, int cnt, int n_entries, int P, int nblk, const int32_t *srow,
                           int n_slots)
{
    int tiles = 0, a = 0, prev = -1;
    while (a < cnt) {
        const int x0 = __ldg(fl + a);
        if (x0 <= prev || x0 >= n_entries) return -1;
        if (!nblk) {
            const int s0 = slot_of(srow, x0);
            if (s0 < 0 || s0 >= n_slots) return -1;
        }
        int lo, hi;
        entry_range(x0, P, nblk, srow, lo, hi);
        const int run_lo = lo;
        prev = x0;
        ++a;
        while (a < cnt) {
            const int x = __ldg(fl + a);
            if (x <= prev || x >= n_entries) return -1;
            if (!nblk) {
                const int s = slot_of(srow, x);
                if (s < 0 || s >= n_slots) return -1;
            }
            int lo2, hi2;
            entry_range(x, P, nblk, srow, lo2, hi2);
            if (lo2 != hi) break;
            hi = hi2;
            prev = x;
            ++a;
        }
        tiles += (hi - run_lo + BN - 1) / BN;
    }
    return tiles;
}

// Walks the attended tokens as runs of contiguous list entries, 128 keys at a time.
struct KvIter {
    const int32_t *fl;
    const int32_t *srow;
    int n, a, P, nblk, pos, end;
    __device__ void init(const int32_t *f, int cnt, int P_, const int32_t *slot_row, int nblk_ = 0)
    {
        fl = f;
        srow = slot_row;
        n = cnt;
        a = 0;
        P = P_;
        nblk = nblk_;
        pos = 0;
        end = 0;
    }
    __device__ void open_run()
    {
        int lo, hi;
        entry_range(__ldg(fl + a), P, nblk, srow, lo, hi);
        ++a;
        while (a < n) {
            int lo2, hi2;
            entry_range(__ldg(fl + a), P, nblk, srow, lo2, hi2);
            if (lo2 != hi) break;
            hi = hi2;
            ++a;
        }
        pos = lo;
        end = hi;
    }
    __device__ void next(int &start, int &nvalid)
    {
        if (pos >= end) open_run();
        start = pos;
        nvalid = min(BN, end - pos);
        pos += BN;
    }
    // skip the first k tiles (whole runs at a time)
    __device__ void skip(int k)
    {
        while (k > 0) {
            if (pos >= end) open_run();
            const int left = (end - pos + BN - 1) / BN;
            if (k >= left) {
                k -= left;
                pos = end;
            } else {
                pos += k * BN;
                k = 0;
            }
        }
    }
};

__device__ __forceinline__ uint32_t mma_n(int nvalid) { return (uint32_t)((nvalid + 15) & ~15); }

// ----------------------------------------------------------------- roles
// Streams the K tiles (IS_K, plus the query tiles first) or the V tiles of the attended
// frames into their ring.  The whole warp runs the loop (its state stays warp-uniform);
// one elected lane issues each copy.  A slot is reused once the MMA warp has released
// it (k_free / v_free: committed after the last MMA that reads the slot).
template <int D, bool IS_K>
__device__ void loader_role(const CUtensorMap *tm_q, const CUtensorMap *tm_kv, const FwdArgs &a, uint32_t sbase,
                            int b, int h, int t, int qt_a, bool has_b, const int32_t *fl, int cnt, int t_off,
                            int n_tiles, const Ctl &ctl)
{
    using C = Cfg<D>;
    constexpr int NSR = IS_K ? C::NSK : C::NSV;
    const Bars<D> bar{sbase + C::SMEM_BAR};
    const uint32_t ring = sbase + (IS_K ? C::SMEM_K : C::SMEM_V);
    if (n_tiles <= 0) return;
    if (IS_K && elect_one()) {
        mbar_arrive_expect_tx(bar.q_full(), C::TILE_BYTES * (has_b ? 2 : 1));
        for (int x = 0; x < (has_b ? 2 : 1); ++x)
#pragma unroll
            for (int kb = 0; kb < C::KBOX; ++kb)
                tma_load_5d(sbase + C::SMEM_Q + x * C::TILE_BYTES + kb * C::BOX_BYTES, tm_q, bar.q_full(), kb * 64,
                            (qt_a + x) * BM, t, h, b);
    }
    __syncwarp();
    // K/V of one (h, t) are re-read by every query tile of the frame: keep them in L2
    const uint64_t policy = l2_policy_evict_last();
    KvIter it;
    it.init(fl, cnt, a.P, a.slots ? a.slots + (int64_t)h * a.T_kv : nullptr, a.nblk);
    it.skip(t_off);
    int j = 0;
    for (; j < n_tiles; ++j) {
        const int s = j % NSR;
        const uint32_t full = IS_K ? bar.k_full(s) : bar.v_full(s);
        if (j >= NSR) {  // one release per use of the slot: exactly one pending phase here
            const uint32_t rel = IS_K ? bar.k_free(s) : bar.v_free(s);
            if (!__all_sync(0xffffffffu, wait_bar(rel, ((j - NSR) / NSR) & 1, ctl))) break;
        }
        int start, nv;
        it.next(start, nv);
        if (elect_one()) {
            mbar_arrive_expect_tx(full, C::TILE_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KBOX; ++kb)
                tma_load_4d(ring + s * C::TILE_BYTES + kb * C::BOX_BYTES, tm_kv, full, kb * 64, start, h, b, policy);
        }
        __syncwarp();
    }
    if (*ctl.abort) {  // let the copies still in flight land before the CTA exits
        if (IS_K) wait_drain(bar.q_full(), 0);
        for (int jj = (j > NSR ? j - NSR : 0); jj < j; ++jj)
            wait_drain(IS_K ? bar.k_full(jj % NSR) : bar.v_full(jj % NSR), (jj / NSR) & 1);
    }
    __syncwarp();
}

// Smem descriptors are built once per CTA; an operand at byte offset `off` from a
// descriptor's base is that descriptor plus off >> 4 (the start address is the low 14
// bits, in 16-byte units; every operand here lies below 256 KB, so nothing carries).
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t off_bytes) { return desc + (off_bytes >> 4); }

template <int D>
__device__ __forceinline__ void issue_s(uint32_t t_s, uint64_t dq, uint64_t dk, uint32_t idesc)
{
    // S[128 x n] = Q[128 x D] K[n x D]^T, both K-major; one MMA per 16 elements of D:
    // +32 bytes inside a 128-byte swizzle row, the next 64 columns one box further on
    if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * Cfg<D>::BOX_BYTES + (kk & 3) * 32;
            mma_ss(t_s, desc_add(dq, off), desc_add(dk, off), idesc, kk > 0);
        }
    }
    __syncwarp();
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t t_o, uint64_t dp, uint64_t dv, uint32_t n, bool accumulate)
{
    // O[128 x D] += P[128 x n] V[n x D]; P K-major in shared memory (like Q), V MN-major
    // (D contiguous): 8-key groups 1024 B apart, 64-wide D blocks one box apart
    constexpr uint32_t idesc = idesc_bf16_f32(BM, D, true);
    const uint32_t steps = n >> 4;
    if (elect_one()) {
#pragma unroll
        for (uint32_t kk = 0; kk < 8; ++kk)
            if (kk < steps)
                mma_ss(t_o, desc_add(dp, (kk >> 2) * Cfg<D>::BOX_BYTES + (kk & 3) * 32), desc_add(dv, kk * 2048),
                       idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
    __syncwarp();
}

// tcgen05.commit from one elected lane of the (converged) MMA warp
__device__ __forceinline__ void commit_one(uint32_t bar)
{
    if (elect_one()) tc_commit(bar);
    __syncwarp();
}

// One warp issues all tensor-core work, in the order
//   S_A(0) S_B(0) | S_A(j+1) P V_A(j) S_B(j+1) P V_B(j) | ...
// While one softmax warpgroup works on its tile, the tensor cores run the other tile's
// next S and P V.  Once the softmax of tile x has handed over P_x(j) it has read S_x(j)
// out, so S_x(j+1) is issued first: the softmax of the next tile starts while P V_x(j)
// still runs, and waits for it (pv_x) only before it overwrites P_x or rescales O_x.
template <int D>
__device__ void mma_role(const FwdArgs &a, uint32_t sbase, uint32_t tmem, int h, bool has_b, const int32_t *fl,
                         int cnt, int t_off, int n_tiles, const Ctl &ctl)
{
    using C = Cfg<D>;
    const Bars<D> bar{sbase + C::SMEM_BAR};
    if (n_tiles <= 0) return;
    const uint64_t dq = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
    const uint64_t dk = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
    const uint64_t dv = sdesc_sw128(sbase + C::SMEM_V, C::BOX_BYTES, 1024);
    const uint64_t dp = sdesc_sw128(sbase + C::SMEM_P, 16, 1024);
    const int nx = has_b ? 2 : 1;
    bool issued = false;
    KvIter it;
    it.init(fl, cnt, a.P, a.slots ? a.slots + (int64_t)h * a.T_kv : nullptr, a.nblk);
    it.skip(t_off);
    int st, nv_cur = 0, nv_next = 0;
    it.next(st, nv_cur);
    if (!__all_sync(0xffffffffu, wait_bar(bar.q_full(), 0, ctl))) goto done;
    if (!__all_sync(0xffffffffu, wait_bar(bar.k_full(0), 0, ctl))) goto done;
    tc_fence_after();
    for (int x = 0; x < nx; ++x) {
        issue_s<D>(tmem + tcol_s(x), desc_add(dq, x * C::TILE_BYTES), dk, idesc_bf16_f32(BM, mma_n(nv_cur), false));
        commit_one(bar.s_full(x));
    }
    commit_one(bar.k_free(0));
    issued = true;
    for (int j = 0; j < n_tiles; ++j) {
        if (j + 1 < n_tiles) it.next(st, nv_next);
        const int sv = j % C::NSV, sk = (j + 1) % C::NSK;
        for (int x = 0; x < nx; ++x) {
            if (!__all_sync(0xffffffffu, wait_bar(bar.p_full(x), j & 1, ctl))) goto done;
            if (j + 1 < n_tiles) {
                if (x == 0 && !__all_sync(0xffffffffu, wait_bar(bar.k_full(sk), ((j + 1) / C::NSK) & 1, ctl)))
                    goto done;
                tc_fence_after();
                issue_s<D>(tmem + tcol_s(x), desc_add(dq, x * C::TILE_BYTES), desc_add(dk, sk * C::TILE_BYTES),
                           idesc_bf16_f32(BM, mma_n(nv_next), false));
                commit_one(bar.s_full(x));
                if (x == nx - 1) commit_one(bar.k_free(sk));  // both tiles' S have read this K slot
            }
            if (x == 0) {
                if (!__all_sync(0xffffffffu, wait_bar(bar.v_full(sv), (j / C::NSV) & 1, ctl))) goto done;
                if (nv_cur & 15) {
                    // P V reads V up to the next multiple of 16 keys, where P is 0; those
                    // few rows hold whatever follows the run in memory (another frame, an
                    // unused cache slot), so they are zeroed first: 0 * (non-finite)
                    // would poison O
                    const int r0 = nv_cur, r1 = (nv_cur + 15) & ~15;
                    const uint32_t vslot = sbase + C::SMEM_V + sv * C::TILE_BYTES;
                    const uint32_t zero[4] = {0u, 0u, 0u, 0u};
                    for (int idx = (int)(threadIdx.x & 31); idx < (r1 - r0) * C::KBOX * 8; idx += 32) {
                        const int r = r0 + idx / (C::KBOX * 8), kb = (idx / 8) % C::KBOX, ch = idx % 8;
                        st_shared_v4(vslot + kb * C::BOX_BYTES + r * 128 + ch * 16, zero);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
            }
            tc_fence_after();
            issue_pv<D>(tmem + tcol_o(x), desc_add(dp, x * C::P_BYTES), desc_add(dv, sv * C::TILE_BYTES),
                        mma_n(nv_cur), j > 0);
            commit_one(bar.pv_x(x));
            if (x == nx - 1) {
                commit_one(bar.v_free(sv));  // both tiles' P V have read this V slot
                // single-phase signal for the epilogues: O of both tiles is complete
                if (j == n_tiles - 1) commit_one(bar.o_final());
            }
        }
        nv_cur = nv_next;
    }
done:
    // (warp-uniform decision: the drain commit below is issued by an elected lane)
    if (__any_sync(0xffffffffu, *ctl.abort != 0) && issued) {  // wait for the tensor cores before TMEM is released
        commit_one(bar.drain());
        wait_drain(bar.drain(), 0);
    }
    __syncwarp();
}

// The tensor-core schedule of a CTA with one query tile (the last, partial tile of a frame
// with an odd number of tiles): the other tile's S and P buffers serve as second buffers,
// S runs two key tiles ahead of the softmax,
//   S(0) S(1) | P V(j) S(j+2) | ...
// so the softmax of tile j+1 starts as soon as it has finished tile j.  S(j+2) goes into
// the buffer the softmax of tile j has read out; P of tile j+2 is written only after
// S(j+2) completes, hence after P V(j).  The softmax rescales O only after P V of the
// previous tile is complete (pv_done).
template <int D>
__device__ void mma_single(const FwdArgs &a, uint32_t sbase, uint32_t tmem, int h, const int32_t *fl, int cnt,
                           int t_off, int n_tiles, const Ctl &ctl)
{
    using C = Cfg<D>;
    const Bars<D> bar{sbase + C::SMEM_BAR};
    if (n_tiles <= 0) return;
    const uint64_t dq = sdesc_sw128(sbase + C::SMEM_Q, 16, 1024);
    const uint64_t dk = sdesc_sw128(sbase + C::SMEM_K, 16, 1024);
    const uint64_t dv = sdesc_sw128(sbase + C::SMEM_V, C::BOX_BYTES, 1024);
    const uint64_t dp = sdesc_sw128(sbase + C::SMEM_P, 16, 1024);
    bool issued = false;
    KvIter it;
    it.init(fl, cnt, a.P, a.slots ? a.slots + (int64_t)h * a.T_kv : nullptr, a.nblk);
    it.skip(t_off);
    int st, nv_j = 0, nv_j1 = 0, nv_j2 = 0;  // valid keys of tiles j, j+1, j+2
    it.next(st, nv_j);
    if (n_tiles > 1) it.next(st, nv_j1);
    if (!__all_sync(0xffffffffu, wait_bar(bar.q_full(), 0, ctl))) goto done;
    for (int j = 0; j < 2 && j < n_tiles; ++j) {
        const int sk = j % C::NSK;
        if (!__all_sync(0xffffffffu, wait_bar(bar.k_full(sk), (j / C::NSK) & 1, ctl))) goto done;
        tc_fence_after();
        issue_s<D>(tmem + tcol_s(j), dq, desc_add(dk, sk * C::TILE_BYTES),
                   idesc_bf16_f32(BM, mma_n(j ? nv_j1 : nv_j), false));
        commit_one(bar.s_full(j));
        commit_one(bar.k_free(sk));
        issued = true;
    }
    for (int j = 0; j < n_tiles; ++j) {
        const int bj = j & 1, sv = j % C::NSV, nvj = nv_j;
        nv_j2 = 0;
        if (j + 2 < n_tiles) it.next(st, nv_j2);
        if (!__all_sync(0xffffffffu, wait_bar(bar.p_full(bj), (j >> 1) & 1, ctl))) goto done;
        if (!__all_sync(0xffffffffu, wait_bar(bar.v_full(sv), (j / C::NSV) & 1, ctl))) goto done;
        if (nvj & 15) {
            // P V reads V up to the next multiple of 16 keys, where P is 0; those few rows
            // hold whatever follows the run in memory, so they are zeroed first
            const int r0 = nvj, r1 = (nvj + 15) & ~15;
            const uint32_t vslot = sbase + C::SMEM_V + sv * C::TILE_BYTES;
            const uint32_t zero[4] = {0u, 0u, 0u, 0u};
            for (int idx = (int)(threadIdx.x & 31); idx < (r1 - r0) * C::KBOX * 8; idx += 32) {
                const int r = r0 + idx / (C::KBOX * 8), kb = (idx / 8) % C::KBOX, ch = idx % 8;
                st_shared_v4(vslot + kb * C::BOX_BYTES + r * 128 + ch * 16, zero);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }
        tc_fence_after();
        issue_pv<D>(tmem + tcol_o(0), desc_add(dp, bj * C::P_BYTES), desc_add(dv, sv * C::TILE_BYTES), mma_n(nvj),
                    j > 0);
        commit_one(bar.pv_done());
        commit_one(bar.v_free(sv));
        if (j == n_tiles - 1) commit_one(bar.o_final());
        if (j + 2 < n_tiles) {
            const int sk = (j + 2) % C::NSK;
            if (!__all_sync(0xffffffffu, wait_bar(bar.k_full(sk), ((j + 2) / C::NSK) & 1, ctl))) goto done;
            tc_fence_after();
            issue_s<D>(tmem + tcol_s(bj), dq, desc_add(dk, sk * C::TILE_BYTES),
                       idesc_bf16_f32(BM, mma_n(nv_j2), false));
            commit_one(bar.s_full(bj));
            commit_one(bar.k_free(sk));
        }
        nv_j = nv_j1;
        nv_j1 = nv_j2;
    }
done:
    if (__any_sync(0xffffffffu, *ctl.abort != 0) && issued) {  // wait for the tensor cores before TMEM is released
        commit_one(bar.drain());
        wait_drain(bar.drain(), 0);
    }
    __syncwarp();
}

// Max of 32 values with 3-input max in a tree (depth 4).
__device__ __forceinline__ float max32(const uint32_t (&r)[32])
{
    float t[11];
#pragma unroll
    for (int k = 0; k < 10; ++k)
        t[k] = fmax3(__uint_as_float(r[3 * k]), __uint_as_float(r[3 * k + 1]), __uint_as_float(r[3 * k + 2]));
    t[10] = fmaxf(__uint_as_float(r[30]), __uint_as_float(r[31]));
    const float u0 = fmax3(t[0], t[1], t[2]), u1 = fmax3(t[3], t[4], t[5]), u2 = fmax3(t[6], t[7], t[8]);
    return fmax3(fmax3(u0, u1, u2), t[9], t[10]);
}

// Columns at or past nv (partial tile) of a loaded 32-column chunk -> -inf.
template <bool FULL>
__device__ __forceinline__ void mask_chunk(int c, int nv, uint32_t (&r)[32])
{
    if (!FULL && (c + 1) * 32 > nv) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= nv) r[i] = __float_as_uint(-INFINITY);
    }
}

// Load 32 columns of this thread's S row; columns at or past nv (partial tile) -> -inf.
template <bool FULL>
__device__ __forceinline__ void load_s_chunk(uint32_t taddr, int c, int nv, uint32_t (&r)[32])
{
    tmem_ld32(taddr + c * 32, r);
    tmem_wait_ld_regs(r);
    if (!FULL && (c + 1) * 32 > nv) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= nv) r[i] = __float_as_uint(-INFINITY);
    }
}

// Eight fp32 partial row sums kept as four pairs, each pair added with one two-lane
// instruction (every lane rounds like a scalar fp32 add, so the sums are those of eight
// scalar accumulators).
struct Acc8 {
    uint64_t v[4] = {0, 0, 0, 0};
    __device__ __forceinline__ void add(int k, float a, float b)
    {
        asm("{\n\t.reg .b64 t;\n\tmov.b64 t, {%1, %2};\n\tadd.rn.f32x2 %0, %0, t;\n\t}"
            : "+l"(v[k])
            : "f"(a), "f"(b));
    }
    __device__ __forceinline__ float get(int i) const
    {
        return __uint_as_float((uint32_t)(v[i >> 1] >> ((i & 1) * 32)));
    }
};

// exp2(s * sl2 - m) of columns 32c..32c+31 -> bf16, stored into this thread's row of the
// P tile in shared memory (K-major, 128-byte swizzle: 64 keys per 16 KB box, 16-byte
// chunk k of row r at chunk position k ^ (r & 7)); row sum into acc
__device__ __forceinline__ void exp_store_chunk(const uint32_t (&r)[32], float sl2, float neg_m, uint32_t p_row,
                                                int row, int c, Acc8 &acc)
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = q * 8 + 2 * i;
            const float p0 = ex2_approx(fmaf(__uint_as_float(r[e]), sl2, neg_m));
            const float p1 = ex2_approx(fmaf(__uint_as_float(r[e + 1]), sl2, neg_m));
            acc.add(i & 3, p0, p1);
            pk[i] = pack_bf16x2(p0, p1);
        }
        const uint32_t chunk = (uint32_t)((c & 1) * 4 + q);
        st_shared_v4(p_row + (c >> 1) * 16384 + ((chunk ^ (uint32_t)(row & 7)) << 4), pk);
    }
}

// exp_store_chunk in two halves: the 16 bf16 pairs of the chunk are formed first and
// stored later, so a wait can sit between them
__device__ __forceinline__ void exp_chunk(const uint32_t (&r)[32], float sl2, float neg_m, uint32_t (&pk)[16],
                                          Acc8 &acc)
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(r[2 * i]), sl2, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(r[2 * i + 1]), sl2, neg_m));
        acc.add(i & 3, p0, p1);
        pk[i] = pack_bf16x2(p0, p1);
    }
}

__device__ __forceinline__ void store_chunk(const uint32_t (&pk)[16], uint32_t p_row, int row, int c)
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t v[4] = {pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]};
        const uint32_t chunk = (uint32_t)((c & 1) * 4 + q);
        st_shared_v4(p_row + (c >> 1) * 16384 + ((chunk ^ (uint32_t)(row & 7)) << 4), v);
    }
}

__device__ __forceinline__ float sum8(const Acc8 &acc)
{
    return ((acc.get(0) + acc.get(1)) + (acc.get(2) + acc.get(3))) +
           ((acc.get(4) + acc.get(5)) + (acc.get(6) + acc.get(7)));
}

// One K/V tile of the online softmax for this thread's query row (thread = TMEM lane):
// S (fp32, TMEM) -> P = exp2(S * scale * log2e - m) as bf16 into shared memory, running
// max m and sum l.  A row keeps a stale max m while a tile's row sum against it stays at
// most RESCALE_LIMIT (every probability is then at most that), so the common case
// streams S through registers 32 columns at a time against the current max.  The first
// tile, and a tile on which any lane of the warp exceeds that sum, take the exact
// two-pass path: row max first, then P against the larger max (S is re-read from TMEM; P
// lives in shared memory), and O is rescaled in place.  FULL: all 128 keys valid.
// pv_first (two-tile CTAs, j > 0): P V of the previous tile may still read P and write O;
// its completion is waited for after the first chunk's exponentials, before any store.
template <int D, bool FULL>
__device__ __forceinline__ bool softmax_tile(uint32_t t_s, uint32_t p_row, int row, uint32_t t_o, int nv, float sl2,
                                             float &m_used, float &l, int j, uint32_t pv_done, uint32_t pv_first,
                                             const Ctl &ctl)
{
    const int nch = FULL ? 4 : (nv + 31) >> 5;
    if (j > 0) {  // streaming pass against the current max
        Acc8 acc;
        const float neg_m = -m_used;
        // two register buffers: the load of chunk c+1 is in flight while chunk c is used
        uint32_t ra[32], rb[32];
        tmem_ld32(t_s, ra);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (FULL || c < nch) {
                uint32_t(&cur)[32] = (c & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
                tmem_wait_ld_regs(cur);
                if (c + 1 < 4 && (FULL || c + 1 < nch)) tmem_ld32(t_s + (c + 1) * 32, nxt);
                mask_chunk<FULL>(c, nv, cur);
                if (c == 0 && pv_first) {
                    uint32_t pk[16];
                    exp_chunk(cur, sl2, neg_m, pk, acc);
                    if (!__all_sync(0xffffffffu, wait_bar(pv_first, (j - 1) & 1, ctl))) return false;
                    tc_fence_after();
                    store_chunk(pk, p_row, row, 0);
                } else {
                    exp_store_chunk(cur, sl2, neg_m, p_row, row, c, acc);
                }
            }
        }
        // a probability above RESCALE_LIMIT (a row max that grew past the stale one by
        // more than 8 in log2 units) makes the tile's row sum exceed it too; a sum above it
        // without such a probability only sends the row through the exact pass a little early
        const float lt = sum8(acc);
        if (!__any_sync(0xffffffffu, lt > RESCALE_LIMIT)) {
            l += lt;
            return true;
        }
    }
    // exact pass: row max over the tile, then P against the new max
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (FULL || c < nch) {
            uint32_t r[32];
            load_s_chunk<FULL>(t_s, c, nv, r);
            mx = fmaxf(mx, max32(r));
        }
    }
    const float m_cand = mx * sl2;
    // (after the streaming pass some probability exceeded 2, so the max has grown)
    const bool resc = m_cand > m_used;
    const float m_new = resc ? m_cand : m_used;
    const float alpha = ex2_approx(m_used - m_new);  // 0 on the first tile, 1 if unchanged
    Acc8 acc;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (FULL || c < nch) {
            uint32_t r[32];
            load_s_chunk<FULL>(t_s, c, nv, r);
            exp_store_chunk(r, sl2, -m_new, p_row, row, c, acc);
        }
    }
    // O must be rescaled before P V of this tile accumulates into it; the warp does it
    // together (tcgen05.ld/st are warp-wide).  In a two-tile CTA P V of the previous tile
    // is already done: the streaming pass waited for it (pv_first).
    if (j > 0 && __any_sync(0xffffffffu, resc)) {
        // (one-tile CTAs run S two tiles ahead: P V of the previous tile may still run)
        if (pv_done) {
            if (!__all_sync(0xffffffffu, wait_bar(pv_done, (j - 1) & 1, ctl))) return false;
            tc_fence_after();
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld_regs(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_o + c * 32, o);
        }
    }
    l = l * alpha + sum8(acc);
    m_used = m_new;
    return true;
}

// Softmax and epilogue of query tile x (0: warps 0-3, 1: warps 4-7), one thread per
// query row.
template <int D>
__device__ void softmax_role(const CUtensorMap *tm_o, const FwdArgs &a, uint8_t *smem, uint32_t sbase,
                             uint32_t tmem, int x, int b, int b_out, int h, int t, int qt, const int32_t *fl,
                             int cnt, int t_off, int n_tiles, bool bad_set, bool one_tile, const Ctl &ctl)
{
    using C = Cfg<D>;
    const Bars<D> bar{sbase + C::SMEM_BAR};
    // 8 flags after the mbarriers (at most 20 x 8 bytes) and before the words at +240
    volatile int32_t *epi_ok = reinterpret_cast<volatile int32_t *>(smem + C::SMEM_BAR + 160) + 4 * x;
    const int row = threadIdx.x & 127;  // query row inside the tile == TMEM lane
    const int warp = (threadIdx.x >> 5) & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t t_o = lane_base + tcol_o(x);
    const float sl2 = a.scale_log2;

    float m_used = -INFINITY;  // running row max (log2 units, scale folded in)
    float l = 0.f;             // running row sum of exp2(s*sl2 - m_used)
    bool alive = true;
    KvIter it;
    it.init(fl, cnt, a.P, a.slots ? a.slots + (int64_t)h * a.T_kv : nullptr, a.nblk);
    it.skip(t_off);
    for (int j = 0; j < n_tiles; ++j) {
        int st, nv;
        it.next(st, nv);
        // S and P buffers: the tile's own, or (a CTA with one query tile) both tiles'
        // buffers in turn, S two tiles ahead.  Either way one pending phase per buffer.
        const int xb = one_tile ? (j & 1) : x;
        const uint32_t par = one_tile ? (uint32_t)(j >> 1) & 1 : (uint32_t)j & 1;
        const uint32_t t_s = lane_base + tcol_s(xb);
        const uint32_t p_row = sbase + C::SMEM_P + xb * C::P_BYTES + row * 128;
        const bool got = wait_bar(bar.s_full(xb), par, ctl);
        if (!__all_sync(0xffffffffu, got)) {
            alive = false;
            break;
        }
        tc_fence_after();
        const uint32_t pvw = one_tile ? bar.pv_done() : 0u;
        const uint32_t pvf = (!one_tile && j > 0) ? bar.pv_x(x) : 0u;
        const bool ok = nv >= BN ? softmax_tile<D, true>(t_s, p_row, row, t_o, nv, sl2, m_used, l, j, pvw, pvf, ctl)
                                 : softmax_tile<D, false>(t_s, p_row, row, t_o, nv, sl2, m_used, l, j, pvw, pvf, ctl);
        if (!ok) {
            alive = false;
            break;
        }
        tmem_wait_st();            // O rescale stores, if any
        fence_proxy_async_smem();  // P written with st.shared is read by the tensor cores
        tc_fence_before();
        __syncwarp();              // one arrival per warp, after all its lanes' writes and fences
        if ((threadIdx.x & 31) == 0 && !((a.debug_flags & SFA_DEBUG_STALL_SOFTMAX) && j == 0))
            mbar_arrive(bar.p_full(xb));
    }

    // ---- epilogue: O / l -> bf16 -> swizzled smem (this tile's Q space) -> TMA store
    bool have = alive;
    if (have && n_tiles > 0) {
        const bool done = wait_bar(bar.o_final(), 0, ctl);
        have = __all_sync(0xffffffffu, done);
    }
    if ((threadIdx.x & 31) == 0) epi_ok[warp] = have ? 1 : 0;
    named_bar_sync(1 + x, BM);
    const bool write = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
    const uint32_t s_o_addr = sbase + C::SMEM_Q + x * C::TILE_BYTES;
    if (write) {
        const float inv_l = n_tiles > 0 ? 1.f / l : 0.f;
        uint8_t *s_o = smem + C::SMEM_Q + x * C::TILE_BYTES;
        if (n_tiles > 0) tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            if (n_tiles > 0) {
                tmem_ld32(t_o + c * 32, o);
                tmem_wait_ld_regs(o);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int col = c * 32 + q * 8;
                const int box = col >> 6, chunk = (col & 63) >> 3;
                uint4 v;
                v.x = pack_bf16x2(__uint_as_float(o[q * 8 + 0]) * inv_l, __uint_as_float(o[q * 8 + 1]) * inv_l);
                v.y = pack_bf16x2(__uint_as_float(o[q * 8 + 2]) * inv_l, __uint_as_float(o[q * 8 + 3]) * inv_l);
                v.z = pack_bf16x2(__uint_as_float(o[q * 8 + 4]) * inv_l, __uint_as_float(o[q * 8 + 5]) * inv_l);
                v.w = pack_bf16x2(__uint_as_float(o[q * 8 + 6]) * inv_l, __uint_as_float(o[q * 8 + 7]) * inv_l);
                *reinterpret_cast<uint4 *>(s_o + box * C::BOX_BYTES + row * 128 + ((chunk ^ (row & 7)) << 4)) = v;
            }
        }
        fence_proxy_async_smem();
    }
    named_bar_sync(1 + x, BM);
    if (write && row == 0) {
#pragma unroll
        for (int kb = 0; kb < C::KBOX; ++kb)
            tma_store_5d(tm_o, s_o_addr + kb * C::BOX_BYTES, kb * 64, qt * BM, t, h, b_out);
        tma_store_commit();
        tma_store_wait_read_all();
    }
    const int p = qt * BM + row;
    if (write && p < a.P) {
        float lse;
        if (bad_set) lse = __int_as_float(0x7fc00000);  // NaN marks a rejected frame list
        else if (n_tiles == 0) lse = -INFINITY;
        else lse = (m_used + log2f(l)) * 0.69314718055994530942f;
        a.lse[((int64_t)(b_out * a.H + h) * a.Tq + t) * a.P + p] = lse;
    }
}

template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    sfa_forward_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ FwdArgs a)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + C::SMEM_BAR;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::SMEM_BAR + 240);
    volatile int32_t *abort_flag = reinterpret_cast<volatile int32_t *>(smem + C::SMEM_BAR + 244);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // a scheduled launch is a programmatic dependent of the schedule kernel: its items (and
    // all that the kernels before that one wrote) are visible after this wait; with partial
    // results, the kernel that merges them may start once every CTA of this grid runs
    if (a.items) pdl_wait();
    if (a.items || gridDim.y > 1) pdl_launch_dependents();

    // work unit: (b, h, t, pair of query tiles), pair fastest so that the tiles sharing
    // one frame's K/V run side by side; the last pair of a frame may hold one tile only
    const int n_pairs = (a.n_qtiles + 1) / 2;
    // work unit and key-tile range: from the CTA's work item (scheduled launch, longest
    // ranges first), or grid y = list set x split: CTA (unit, y) takes list set y / n_split
    // and key-tile range y mod n_split of it
    int x, li, split, n_split, slice;
    if (a.items) {
        const int2 w = a.items[blockIdx.x];
        x = w.x;
        li = w.y & 1;
        split = (w.y >> 1) & 255;
        n_split = w.y >> 9;
        slice = li ? a.k_first + split : split;
    } else {
        x = blockIdx.x;
        n_split = gridDim.y / a.n_lists;
        li = blockIdx.y / n_split;
        split = blockIdx.y - li * n_split;
        slice = blockIdx.y;
    }
    const int qt_a = 2 * (x % n_pairs);
    const bool has_b = qt_a + 1 < a.n_qtiles;
    x /= n_pairs;
    const int t = x % a.Tq;
    x /= a.Tq;
    const int h = x % a.H;
    const int b = x / a.H;
    // the unit's list: frames of (h, t), or key blocks of (b, h, t, query block = pair)
    const int64_t list = a.nblk ? ((((int64_t)b * a.H + h) * a.Tq + t) * n_pairs + qt_a / 2) : (int64_t)h * a.Tq + t;
    const int32_t *fl = (li ? a.frames2 : a.frames) + list * a.Amax;
    const int cnt = __ldg((li ? a.counts2 : a.counts) + list);
    int n_all = (cnt >= 0 && cnt <= a.Amax)
                    ? count_tiles(fl, cnt, a.nblk ? a.T_kv * a.nblk : a.T_kv, a.P, a.nblk,
                                  a.slots ? a.slots + (int64_t)h * a.T_kv : nullptr, a.n_slots)
                    : -1;
    const bool bad_set = n_all < 0;
    if (bad_set) n_all = 0;
    // split-KV: CTA (unit, split) takes the unit's key tiles [t_off, t_off + n_tiles) and,
    // with more than one slice, writes a partial result into its slice of the output
    // (batch index b_out)
    const int t_off = (int)(((int64_t)n_all * split) / n_split);
    int n_tiles = (int)(((int64_t)n_all * (split + 1)) / n_split) - t_off;
    const int b_out = slice * a.B + b;
    volatile int32_t *skip = reinterpret_cast<volatile int32_t *>(smem + C::SMEM_BAR + 248);

    if (threadIdx.x == 0) {
        const Bars<D> bar{bars};
        for (int i = 0; i < Bars<D>::COUNT; ++i) mbar_init(bars + 8 * i, 1);
        mbar_init(bar.p_full(0), BM / 32);  // P full: every softmax warp of the tile arrives
        mbar_init(bar.p_full(1), BM / 32);
        *abort_flag = 0;
        // once a CTA has timed out, the ones that start later skip their work
        *skip = (a.status && *reinterpret_cast<volatile int32_t *>(a.status) == SFA_ERR_TIMEOUT) ? 1 : 0;
        fence_mbar_init();
        if (bad_set && split == 0) report(a.status, SFA_ERR_BAD_SET);
    }
    if (warp == K_LOAD_WARP && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Ctl ctl{abort_flag, a.status, a.timeout_ns};
    const bool skipped = *skip != 0;
    if (skipped) n_tiles = 0;

    if (warp == K_LOAD_WARP) {
        loader_role<D, true>(&tm_q, &tm_k, a, sbase, b, h, t, qt_a, has_b, fl, cnt, t_off, n_tiles, ctl);
    } else if (warp == V_LOAD_WARP) {
        loader_role<D, false>(&tm_q, &tm_v, a, sbase, b, h, t, qt_a, has_b, fl, cnt, t_off, n_tiles, ctl);
    } else if (warp == MMA_WARP) {
        if (has_b) mma_role<D>(a, sbase, tmem, h, has_b, fl, cnt, t_off, n_tiles, ctl);
        else mma_single<D>(a, sbase, tmem, h, fl, cnt, t_off, n_tiles, ctl);
    } else if (warp < 8) {
        const int xt = warp >> 2;  // query tile of this softmax warpgroup
        if (!skipped && (xt == 0 || has_b))
            softmax_role<D>(&tm_o, a, smem, sbase, tmem, xt, b, b_out, h, t, qt_a + xt, fl, cnt, t_off, n_tiles,
                            bad_set, !has_b, ctl);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ----------------------------------------------------------------- scheduled launches
// A scheduled launch runs one CTA per work item: (list set, unit, key-tile range), the
// ranges of list set l being k_l equal parts of the unit's key tiles.  The items are
// ordered longest range first, so that the hardware block scheduler, which hands CTAs to
// SMs in index order as they free up, runs a longest-processing-time-first schedule: long
// units start in the first wave and short ones fill the tail.  Ranges are ranked by a
// coarse length class (an octave), and inside a class the natural order is kept (a stable
// counting sort): units of similar length stay in (batch, head, frame) order, so the CTAs
// that read the same keys (the pairs of one list, the frames of one head, the query blocks
// of one frame) run side by side and find them in L2.  Finer classes measured worse: the
// key-block lists of one frame (100 to 115 key tiles) fell into two quarter-octave classes,
// each head's keys were then read twice from HBM, and the launch took 1.0 ms against 0.56.
constexpr int SCHED_THREADS = 1024;
constexpr int SCHED_BINS = 32;  // length classes: floor(log2(range))
constexpr int SCHED_CACHE = 8192;  // entries whose class the first pass keeps for the second

struct SchedArgs {
    const int32_t *frames[2];
    const int32_t *counts[2];
    int32_t k[2];      // key-tile ranges per unit of each list set
    int32_t n_lists;   // list sets (1 or 2)
    int32_t B, H, Tq, T_kv, P, Amax, nblk, n_pairs, n_slots;
    const int32_t *slots;
    int2 *items;
};

// Key tiles of entry e of list set li (0 for a malformed list: the forward CTA reports it).
__device__ int sched_len(const SchedArgs &s, int li, int e)
{
    const int32_t *fl = s.frames[li] + (int64_t)e * s.Amax;
    const int cnt = __ldg(s.counts[li] + e);
    if (cnt < 0 || cnt > s.Amax) return 0;
    const int h = s.nblk ? (e / (s.Tq * s.n_pairs)) % s.H : e / s.Tq;
    const int32_t *srow = s.slots ? s.slots + (int64_t)h * s.T_kv : nullptr;
    const int n = count_tiles(fl, cnt, s.nblk ? s.T_kv * s.nblk : s.T_kv, s.P, s.nblk, srow, s.n_slots);
    return n > 0 ? n : 0;
}

// Length class of a range of `len` key tiles: higher runs first.
__device__ __forceinline__ int sched_bin(int len) { return len <= 1 ? 0 : 31 - __clz(len); }

__global__ void __launch_bounds__(SCHED_THREADS) schedule_kernel(const __grid_constant__ SchedArgs s)
{
    pdl_launch_dependents();  // the forward kernel's CTAs may take their SMs and wait for the items
    constexpr int NW = SCHED_THREADS / 32;
    __shared__ int bin_start[SCHED_BINS];     // first item of each class (descending class order)
    __shared__ int carry[SCHED_BINS];         // items of each class placed by earlier chunks
    __shared__ int wcount[NW][SCHED_BINS];    // items of each class per warp, this chunk
    __shared__ uint8_t cls[SCHED_CACHE];      // class of the first SCHED_CACHE entries
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // entries: frame lists per (h, t), or key-block lists per unit; units per entry
    const int per_set = s.nblk ? s.B * s.H * s.Tq * s.n_pairs : s.H * s.Tq;
    const int fan = s.nblk ? 1 : s.B * s.n_pairs;
    const int n_entries = per_set * s.n_lists;
    if (tid < SCHED_BINS) {
        bin_start[tid] = 0;
        carry[tid] = 0;
    }
    __syncthreads();
    for (int e = tid; e < n_entries; e += SCHED_THREADS) {
        const int li = e / per_set, k = s.k[li];
        const int bin = sched_bin((sched_len(s, li, e - li * per_set) + k - 1) / k);
        if (e < SCHED_CACHE) cls[e] = (uint8_t)bin;
        atomicAdd(&bin_start[bin], fan * k);
    }
    __syncthreads();
    if (tid == 0) {  // exclusive prefix in descending class order
        int acc = 0;
        for (int b = SCHED_BINS - 1; b >= 0; --b) {
            const int v = bin_start[b];
            bin_start[b] = acc;
            acc += v;
        }
    }
    __syncthreads();
    // stable placement, SCHED_THREADS entries per chunk in entry order: an entry's items go
    // after those of every earlier entry of its class
    for (int c0 = 0; c0 < n_entries; c0 += SCHED_THREADS) {
        const int e = c0 + tid;
        const bool on = e < n_entries;
        int li = 0, le = 0, k = 1, bin = -1;
        if (on) {
            li = e / per_set;
            le = e - li * per_set;
            k = s.k[li];
            bin = e < SCHED_CACHE ? cls[e] : sched_bin((sched_len(s, li, le) + k - 1) / k);
        }
        for (int i = tid; i < NW * SCHED_BINS; i += SCHED_THREADS) (&wcount[0][0])[i] = 0;
        __syncthreads();
        // lanes of this warp in the same class, before this lane: their items come first
        // (an entry of list set l has fan * k_l items)
        const unsigned same = __match_any_sync(0xffffffffu, bin);
        const unsigned in_set1 = __ballot_sync(0xffffffffu, on && li == 1);
        const unsigned lt = (1u << lane) - 1u;
        const int k0 = s.k[0], k1 = s.n_lists == 2 ? s.k[1] : 0;
        const int before = fan * (k0 * __popc(same & lt & ~in_set1) + k1 * __popc(same & lt & in_set1));
        if (on && __popc(same & lt) == 0)  // the class's first lane in this warp
            wcount[warp][bin] = fan * (k0 * __popc(same & ~in_set1) + k1 * __popc(same & in_set1));
        __syncthreads();
        if (on) {
            int off = bin_start[bin] + carry[bin] + before;
            for (int w = 0; w < warp; ++w) off += wcount[w][bin];
            for (int sp = 0; sp < k; ++sp) {
                const int tag = li | (sp << 1) | (k << 9);
                if (s.nblk) {
                    s.items[off++] = make_int2(le, tag);
                } else {
                    const int h = le / s.Tq, t = le - h * s.Tq;
                    for (int b = 0; b < s.B; ++b)
                        for (int pr = 0; pr < s.n_pairs; ++pr)
                            s.items[off++] = make_int2(((b * s.H + h) * s.Tq + t) * s.n_pairs + pr, tag);
                }
            }
        }
        __syncthreads();
        if (tid < SCHED_BINS) {
            int add = 0;
            for (int w = 0; w < NW; ++w) add += wcount[w][tid];
            carry[tid] += add;
        }
        __syncthreads();
    }
}

// ----------------------------------------------------------------- host side
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

// bf16 tensor map, 128-byte swizzle, box = 64 elements x 128 rows (x 1 ...)
bool encode(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t box[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        es[i] = 1;
        box[i] = i == 0 ? 64 : (i == 1 ? 128 : 1);
    }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), gd, gs, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool stride_ok(const int64_t *s, int d)
{
    for (int i = 0; i < 3; ++i)
        if (s[i] <= 0 || s[i] % 8 || s[i] >= ((int64_t)1 << 38)) return false;
    return s[2] >= d;
}

// Scheduled launch: key-tile ranges per unit of each list set, and room for the work items.
struct Schedule {
    int k0, k1;
    int2 *items;
};

// Forward launch.  n_split == 1: O and LSE go to the caller's buffers.  n_split > 1:
// every unit's key tiles are split into n_split ranges, CTA (unit, split) writes its
// partial O / LSE into the workspace slices [split][B][H][Tq*P][d] (bf16, contiguous) and
// [split][B][H][Tq*P] (fp32), and a k-way LSE merge writes the caller's O and LSE.  With a
// schedule the list sets take k0 and k1 ranges, one CTA per work item, longest first.
template <int D>
sfa_status launch(const sfa_attn_desc *d, const void *q, const void *k, const void *v, const int32_t *frames,
                  const int32_t *counts, void *o, float *lse, int32_t *dev_status, cudaStream_t stream,
                  int n_split = 1, void *ws_o = nullptr, float *ws_lse = nullptr, const int32_t *slots = nullptr,
                  int n_slots = 0, int nblk = 0, const int32_t *frames2 = nullptr, const int32_t *counts2 = nullptr,
                  void *o_first = nullptr, float *lse_first = nullptr, const Schedule *sched = nullptr)
{
    using C = Cfg<D>;
    const int n_lists = frames2 ? 2 : 1;
    // partial outputs (1: straight to o / lse)
    const int slices = sched ? sched->k0 + (n_lists == 2 ? sched->k1 : 0) : n_lists * n_split;
    const int k_first = sched ? sched->k0 : n_split;
    CUtensorMap tq, tk, tv, to;
    const int kv_frames = slots ? n_slots : d->T_kv;  // frames held by the K/V buffers
    const uint64_t P = d->P, Tq = d->Tq, Lkv = (uint64_t)kv_frames * d->P;
    {
        const uint64_t dims[5] = {(uint64_t)D, P, Tq, (uint64_t)d->H, (uint64_t)d->B};
        const uint64_t st[4] = {(uint64_t)d->q_stride[2] * 2, P * d->q_stride[2] * 2, (uint64_t)d->q_stride[1] * 2,
                                (uint64_t)d->q_stride[0] * 2};
        if (!encode(&tq, q, 5, dims, st)) return SFA_ERR_UNSUPPORTED;
        if (slices == 1) {
            const uint64_t so[4] = {(uint64_t)d->o_stride[2] * 2, P * d->o_stride[2] * 2,
                                    (uint64_t)d->o_stride[1] * 2, (uint64_t)d->o_stride[0] * 2};
            if (!encode(&to, o, 5, dims, so)) return SFA_ERR_UNSUPPORTED;
        } else {
            const uint64_t Lq = Tq * P;
            const uint64_t dims_w[5] = {(uint64_t)D, P, Tq, (uint64_t)d->H, (uint64_t)d->B * slices};
            const uint64_t sw[4] = {(uint64_t)D * 2, P * D * 2, Lq * D * 2, (uint64_t)d->H * Lq * D * 2};
            if (!encode(&to, ws_o, 5, dims_w, sw)) return SFA_ERR_UNSUPPORTED;
        }
    }
    {
        const uint64_t dims[4] = {(uint64_t)D, Lkv, (uint64_t)d->H, (uint64_t)d->B};
        const uint64_t sk[3] = {(uint64_t)d->k_stride[2] * 2, (uint64_t)d->k_stride[1] * 2,
                                (uint64_t)d->k_stride[0] * 2};
        const uint64_t sv[3] = {(uint64_t)d->v_stride[2] * 2, (uint64_t)d->v_stride[1] * 2,
                                (uint64_t)d->v_stride[0] * 2};
        if (!encode(&tk, k, 4, dims, sk)) return SFA_ERR_UNSUPPORTED;
        if (!encode(&tv, v, 4, dims, sv)) return SFA_ERR_UNSUPPORTED;
    }
    FwdArgs a;
    a.B = d->B;
    a.H = d->H;
    a.Tq = d->Tq;
    a.T_kv = d->T_kv;
    a.P = d->P;
    a.Amax = d->Amax;
    a.n_qtiles = (d->P + BM - 1) / BM;
    a.scale_log2 = d->scale * 1.4426950408889634f;
    a.frames = frames;
    a.counts = counts;
    a.slots = slots;
    a.n_slots = kv_frames;
    a.nblk = nblk;
    a.lse = slices == 1 ? lse : ws_lse;
    a.frames2 = frames2;
    a.counts2 = counts2;
    a.n_lists = n_lists;
    a.items = sched ? sched->items : nullptr;
    a.k_first = k_first;
    a.status = dev_status;
    a.timeout_ns = (uint64_t)(d->timeout_us ? d->timeout_us : DEFAULT_TIMEOUT_US) * 1000;
    a.debug_flags = d->debug_flags;

    const int64_t grid = (int64_t)d->B * d->H * d->Tq * ((a.n_qtiles + 1) / 2);
    if (cudaFuncSetAttribute(sfa_forward_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return SFA_ERR_CUDA;
    if (sched) {
        SchedArgs sa;
        sa.frames[0] = frames;
        sa.counts[0] = counts;
        sa.frames[1] = frames2 ? frames2 : frames;
        sa.counts[1] = counts2 ? counts2 : counts;
        sa.k[0] = sched->k0;
        sa.k[1] = n_lists == 2 ? sched->k1 : 0;
        sa.n_lists = n_lists;
        sa.B = d->B;
        sa.H = d->H;
        sa.Tq = d->Tq;
        sa.T_kv = d->T_kv;
        sa.P = d->P;
        sa.Amax = d->Amax;
        sa.nblk = nblk;
        sa.n_pairs = (a.n_qtiles + 1) / 2;
        sa.n_slots = kv_frames;
        sa.slots = slots;
        sa.items = sched->items;
        schedule_kernel<<<1, SCHED_THREADS, 0, stream>>>(sa);
        sfa_status st0 = launch_status();
        if (st0 != SFA_OK) return st0;
        const int64_t n_items = grid * (sched->k0 + (n_lists == 2 ? sched->k1 : 0));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)n_items, 1);
        cfg.blockDim = dim3(NUM_THREADS);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, sfa_forward_kernel<D>, tq, tk, tv, to, a) != cudaSuccess) return SFA_ERR_CUDA;
    } else {
        sfa_forward_kernel<D><<<dim3((unsigned)grid, (unsigned)slices), NUM_THREADS, C::SMEM_BYTES, stream>>>(
            tq, tk, tv, to, a);
    }
    sfa_status st = launch_status();
    if (st != SFA_OK || slices == 1) return st;
    const int64_t Lq = (int64_t)d->Tq * d->P;
    return launch_lse_combine((int64_t)d->B * d->H * Lq, slices, D, d->H, Lq, ws_o, ws_lse, o, d->o_stride, lse,
                              stream, n_lists == 2 ? k_first : 0, o_first, lse_first);
}

size_t split_ws_o_bytes(const sfa_attn_desc *d, int n_split)
{
    const size_t rows = (size_t)d->B * d->H * d->Tq * d->P;
    return ((size_t)n_split * rows * d->d * 2 + 255) / 256 * 256;
}

size_t split_ws_bytes(const sfa_attn_desc *d, int n_split)
{
    const size_t rows = (size_t)d->B * d->H * d->Tq * d->P;
    return split_ws_o_bytes(d, n_split) + ((size_t)n_split * rows * 4 + 255) / 256 * 256;
}

// ----------------------------------------------------------------- automatic split
// n_split = 0 asks for a scheduled launch with the key-tile ranges per unit chosen here.
// The host does not see the lists (they live on the device), so the choice uses Amax as
// every unit's length (an upper bound) and models the launch as waves of equal pieces,
// each a range plus a fixed prologue / epilogue cost, plus the merge of the partials;
// the schedule kernel then orders the real ranges longest first.
constexpr double SCHED_OVERHEAD_TILES = 3.0;  // Q load, pipeline fill, epilogue of one CTA, in key tiles
// the same for the ranges of a two-list launch: fitted to a sweep of the history branch's
// range count on the LSE-merge workload (12 heads x 7 query-tile pairs, lists of 2 and 12
// frames; 4, 5, 6, 7, 8, 10 ranges measured 0.263, 0.290, 0.271, 0.286, 0.294, 0.300 ms),
// whose order the 3-tile figure does not reproduce (it picked 6)
constexpr double DUAL_OVERHEAD_TILES = 16.0;
constexpr double STEP_US = 2.4;               // one key tile of a CTA (both query tiles), measured
constexpr double HBM_BYTES_PER_US = 6.5e6;

int sm_count()
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

// Ranges per unit (k0 for the first list set, k1 for the second) of a scheduled launch.
void auto_splits(const sfa_attn_desc *d, int n_lists, int nblk, int &k0, int &k1)
{
    const int sms = sm_count();
    const int n_qt = (d->P + BM - 1) / BM;
    const double units = (double)d->B * d->H * d->Tq * ((n_qt + 1) / 2);
    const double len = nblk ? (double)d->Amax : (double)d->Amax * n_qt;  // key tiles per unit, at most
    const int cap = d->d / 8;                                           // partial slices the merge takes
    const double slice_bytes = (double)d->B * d->H * d->Tq * d->P * (2.0 * d->d + 4.0);
    auto cost = [&](int pieces_per_unit, int longest_k, int slices, double overhead = SCHED_OVERHEAD_TILES) {
        const double piece = std::ceil(len / longest_k) + overhead;
        const double waves = std::ceil(units * pieces_per_unit / sms);
        const double merge = slices > 1 ? (slices + 1) * slice_bytes / HBM_BYTES_PER_US : 0.0;
        return waves * piece * STEP_US + merge;
    };
    k1 = 0;
    if (n_lists == 1) {
        k0 = 1;
        if (units >= 8.0 * sms) return;  // many full waves: splitting only adds merge traffic
        // key-block lists: measured on the hsa workload, their ranges cost more than they
        // recover (0.67 ms at 2 ranges, 1.20 at 4, 0.56 unsplit), so they keep one range
        // unless the grid fills less than half the SMs
        if (nblk && units >= 0.5 * sms) return;
        double best = cost(1, 1, 1);
        for (int k = 2; k <= cap; ++k) {
            const double c = cost(k, k, k);
            if (c < best) {
                best = c;
                k0 = k;
            }
        }
        return;
    }
    // two list sets sharing Amax: the first (local) branch is the short one and keeps one
    // range per unit; the second (history) branch is split
    k0 = 1;
    k1 = 1;
    double best = cost(2, 1, 2, DUAL_OVERHEAD_TILES);
    for (int k = 2; k + 1 <= cap; ++k) {
        const double c = cost(1 + k, k, 1 + k, DUAL_OVERHEAD_TILES);
        if (c < best) {
            best = c;
            k1 = k;
        }
    }
}

size_t sched_items_bytes(const sfa_attn_desc *d, int pieces_per_unit)
{
    const size_t grid = (size_t)d->B * d->H * d->Tq * (((d->P + BM - 1) / BM + 1) / 2);
    return (grid * pieces_per_unit * sizeof(int2) + 255) / 256 * 256;
}

// Workspace of a scheduled launch: the partial slices (when there are several), then the items.
size_t sched_ws_bytes(const sfa_attn_desc *d, int k0, int k1)
{
    const int slices = k0 + k1;
    return (slices > 1 ? split_ws_bytes(d, slices) : 0) + sched_items_bytes(d, slices);
}

sfa_status check_desc(const sfa_attn_desc *d)
{
    if (!d) return SFA_ERR_INVALID_ARG;
    if (d->B < 0 || d->H < 1 || d->Tq < 1 || d->T_kv < 1 || d->P < 1 || d->Amax < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return SFA_ERR_UNSUPPORTED;
    if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return SFA_ERR_INVALID_ARG;
    if ((int64_t)d->Tq * d->P >= ((int64_t)1 << 31) || (int64_t)d->T_kv * d->P >= ((int64_t)1 << 31))
        return SFA_ERR_INVALID_ARG;
    const int64_t grid = (int64_t)d->B * d->H * d->Tq * ((d->P + BM - 1) / BM);
    if (grid >= ((int64_t)1 << 31)) return SFA_ERR_INVALID_ARG;
    return SFA_OK;
}

sfa_status check_buffers(const sfa_attn_desc *d, const void *q, const void *k, const void *v, const int32_t *frames,
                         const int32_t *counts, const void *o, const float *lse)
{
    if (!q || !k || !v || !o || !lse || !frames || !counts) return SFA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, o})
        if (reinterpret_cast<uintptr_t>(p) % 16) return SFA_ERR_INVALID_ARG;
    if (!stride_ok(d->q_stride, d->d) || !stride_ok(d->k_stride, d->d) || !stride_ok(d->v_stride, d->d) ||
        !stride_ok(d->o_stride, d->d))
        return SFA_ERR_INVALID_ARG;
    return SFA_OK;
}

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_forward(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                  const int32_t *frames, const int32_t *counts, void *o, float *lse,
                                  int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, frames, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s)
                       : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s);
}

extern "C" sfa_status sfa_forward_split_workspace(const sfa_attn_desc *d, int32_t n_split, size_t *bytes)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (!bytes || n_split < 0 || n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (n_split == 0) {
        int k0, k1;
        auto_splits(d, 1, 0, k0, k1);
        *bytes = sched_ws_bytes(d, k0, 0);
        return SFA_OK;
    }
    *bytes = n_split == 1 ? 0 : split_ws_bytes(d, n_split);
    return SFA_OK;
}

extern "C" sfa_status sfa_forward_split_plan(const sfa_attn_desc *d, int32_t n_lists, int32_t key_blocks,
                                             int32_t *k_first, int32_t *k_second)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (!k_first || (n_lists != 1 && n_lists != 2) || (key_blocks && n_lists != 1)) return SFA_ERR_INVALID_ARG;
    int k0, k1;
    auto_splits(d, n_lists, key_blocks ? (d->P + KEY_BLOCK - 1) / KEY_BLOCK : 0, k0, k1);
    *k_first = k0;
    if (k_second) *k_second = k1;
    return SFA_OK;
}

extern "C" sfa_status sfa_forward_split(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                        const int32_t *frames, const int32_t *counts, void *o, float *lse,
                                        int32_t n_split, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (n_split < 0 || n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, frames, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    if (n_split == 0) {  // scheduled: ranges chosen here, longest first
        Schedule sc;
        auto_splits(d, 1, 0, sc.k0, sc.k1);
        if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < sched_ws_bytes(d, sc.k0, 0))
            return SFA_ERR_INVALID_ARG;
        if (sc.k0 == 1)  // one range per unit: the plain launch (ordering alone measured no gain)
            return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s)
                               : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s);
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        sc.items = reinterpret_cast<int2 *>(ws + (sc.k0 > 1 ? split_ws_bytes(d, sc.k0) : 0));
        float *ws_lse = reinterpret_cast<float *>(ws + split_ws_o_bytes(d, sc.k0));
        void *ws_o = sc.k0 > 1 ? workspace : nullptr;
        if (sc.k0 == 1) ws_lse = nullptr;
        return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s, sc.k0, ws_o, ws_lse,
                                         nullptr, 0, 0, nullptr, nullptr, nullptr, nullptr, &sc)
                           : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s, sc.k0, ws_o, ws_lse,
                                        nullptr, 0, 0, nullptr, nullptr, nullptr, nullptr, &sc);
    }
    if (n_split == 1)
        return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s)
                           : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s);
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < split_ws_bytes(d, n_split))
        return SFA_ERR_INVALID_ARG;
    float *ws_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) + split_ws_o_bytes(d, n_split));
    return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s, n_split, workspace, ws_lse)
                       : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s, n_split, workspace, ws_lse);
}

// ------------------------------------------------------------------------------------
// Host buffers in, host buffers out: the copies and the attention as one pipeline.
// The (batch, head-group) chunks run in order: the copy of chunk i+1 to the device (one
// stream), the attention of chunk i (two streams in turn, so the last wave of one kernel
// overlaps the first of the next) and the copy of chunk i-1 back (a third stream) overlap.
// ------------------------------------------------------------------------------------
namespace sfa {
namespace {

struct HostLayout {
    size_t q, k, v, o, lse, total;
};

HostLayout host_layout(const sfa_attn_desc *d)
{
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t bh = (size_t)d->B * d->H, lq = (size_t)d->Tq * d->P, lk = (size_t)d->T_kv * d->P;
    HostLayout w;
    w.q = 0;
    w.k = up(bh * lq * d->d * 2);
    w.v = w.k + up(bh * lk * d->d * 2);
    w.o = w.v + up(bh * lk * d->d * 2);
    w.lse = w.o + up(bh * lq * d->d * 2);
    w.total = w.lse + up(bh * lq * 4);
    return w;
}

// RAII set of the call's streams and events (released when the call returns; work still
// queued on a destroyed stream completes normally)
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr, run[2] = {nullptr, nullptr};
    cudaEvent_t start = nullptr, e_in = nullptr, e_run[2] = {nullptr, nullptr}, end[4] = {};
    bool ok = true;
    HostPipe()
    {
        for (cudaStream_t *st : {&in, &out, &run[0], &run[1]})
            ok = ok && cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) == cudaSuccess;
        for (cudaEvent_t *ev : {&start, &e_in, &e_run[0], &e_run[1], &end[0], &end[1], &end[2], &end[3]})
            ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
    }
    ~HostPipe()
    {
        for (cudaEvent_t ev : {start, e_in, e_run[0], e_run[1], end[0], end[1], end[2], end[3]})
            if (ev) cudaEventDestroy(ev);
        for (cudaStream_t st : {in, out, run[0], run[1]})
            if (st) cudaStreamDestroy(st);
    }
};

}  // namespace
}  // namespace sfa

extern "C" sfa_status sfa_forward_host_workspace(const sfa_attn_desc *d, size_t *bytes)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (!bytes) return SFA_ERR_INVALID_ARG;
    *bytes = host_layout(d).total;
    return SFA_OK;
}

extern "C" sfa_status sfa_forward_host(const sfa_attn_desc *d, const void *q_host, const void *k_host,
                                       const void *v_host, const int32_t *frames, const int32_t *counts,
                                       void *o_host, float *lse_host, int32_t n_chunks, void *workspace,
                                       size_t workspace_bytes, int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (n_chunks < 1) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!q_host || !k_host || !v_host || !o_host || !lse_host || !frames || !counts) return SFA_ERR_INVALID_ARG;
    const HostLayout w = host_layout(d);
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < w.total)
        return SFA_ERR_INVALID_ARG;
    const int64_t lq = (int64_t)d->Tq * d->P, lk = (int64_t)d->T_kv * d->P, D = d->d;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *q = ws + w.q, *k = ws + w.k, *v = ws + w.v, *o = ws + w.o;
    float *lse = reinterpret_cast<float *>(ws + w.lse);
    const uint8_t *qh = static_cast<const uint8_t *>(q_host), *kh = static_cast<const uint8_t *>(k_host),
                  *vh = static_cast<const uint8_t *>(v_host);
    uint8_t *oh = static_cast<uint8_t *>(o_host);
    cudaStream_t main = as_cuda(stream);
    HostPipe pp;
    if (!pp.ok) return SFA_ERR_CUDA;
    // every side stream starts after the work already queued on the caller's stream
    if (cudaEventRecord(pp.start, main) != cudaSuccess) return SFA_ERR_CUDA;
    for (cudaStream_t sx : {pp.in, pp.out, pp.run[0], pp.run[1]})
        if (cudaStreamWaitEvent(sx, pp.start, 0) != cudaSuccess) return SFA_ERR_CUDA;
    // chunks: per batch entry, groups of heads (contiguous in the [B][H][L][d] layout)
    auto enqueue = [&]() -> sfa_status {
        const int per_b = std::max(1, std::min<int>(d->H, n_chunks >= d->B ? n_chunks / d->B : 1));
        int c = 0;
        for (int b = 0; b < d->B; ++b) {
            for (int g = 0; g < per_b; ++g, ++c) {
                const int h0 = (int)((int64_t)d->H * g / per_b), h1 = (int)((int64_t)d->H * (g + 1) / per_b);
                if (h1 == h0) continue;
                const int64_t hq = ((int64_t)b * d->H + h0) * lq, hk = ((int64_t)b * d->H + h0) * lk;
                const int64_t nq = (int64_t)(h1 - h0) * lq, nk = (int64_t)(h1 - h0) * lk;
                const size_t bq = (size_t)nq * D * 2, bk = (size_t)nk * D * 2;
                if (cudaMemcpyAsync(q + hq * D * 2, qh + hq * D * 2, bq, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                    cudaMemcpyAsync(k + hk * D * 2, kh + hk * D * 2, bk, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                    cudaMemcpyAsync(v + hk * D * 2, vh + hk * D * 2, bk, cudaMemcpyHostToDevice, pp.in) != cudaSuccess ||
                    cudaEventRecord(pp.e_in, pp.in) != cudaSuccess)
                    return SFA_ERR_CUDA;
                cudaStream_t run = pp.run[c & 1];
                if (cudaStreamWaitEvent(run, pp.e_in, 0) != cudaSuccess) return SFA_ERR_CUDA;
                sfa_attn_desc cd = *d;
                cd.B = 1;
                cd.H = h1 - h0;
                cd.q_stride[0] = cd.o_stride[0] = (int64_t)cd.H * lq * D;
                cd.q_stride[1] = cd.o_stride[1] = lq * D;
                cd.q_stride[2] = cd.o_stride[2] = D;
                cd.k_stride[0] = cd.v_stride[0] = (int64_t)cd.H * lk * D;
                cd.k_stride[1] = cd.v_stride[1] = lk * D;
                cd.k_stride[2] = cd.v_stride[2] = D;
                const int32_t *fr = frames + (int64_t)h0 * d->Tq * d->Amax, *cn = counts + (int64_t)h0 * d->Tq;
                st = D == 128 ? launch<128>(&cd, q + hq * D * 2, k + hk * D * 2, v + hk * D * 2, fr, cn, o + hq * D * 2,
                                            lse + hq, dev_status, run)
                              : launch<64>(&cd, q + hq * D * 2, k + hk * D * 2, v + hk * D * 2, fr, cn, o + hq * D * 2,
                                           lse + hq, dev_status, run);
                if (st != SFA_OK) return st;
                if (cudaEventRecord(pp.e_run[c & 1], run) != cudaSuccess ||
                    cudaStreamWaitEvent(pp.out, pp.e_run[c & 1], 0) != cudaSuccess ||
                    cudaMemcpyAsync(oh + hq * D * 2, o + hq * D * 2, bq, cudaMemcpyDeviceToHost, pp.out) != cudaSuccess ||
                    cudaMemcpyAsync(lse_host + hq, lse + hq, (size_t)nq * 4, cudaMemcpyDeviceToHost, pp.out) !=
                        cudaSuccess)
                    return SFA_ERR_CUDA;
            }
        }
        return SFA_OK;
    };
    const sfa_status queued = enqueue();
    // the caller's stream waits for the whole pipeline, like a single kernel on it (also
    // after an error, for whatever was queued)
    int i = 0;
    sfa_status joined = SFA_OK;
    for (cudaStream_t sx : {pp.in, pp.out, pp.run[0], pp.run[1]}) {
        if (cudaEventRecord(pp.end[i], sx) != cudaSuccess || cudaStreamWaitEvent(main, pp.end[i], 0) != cudaSuccess)
            joined = SFA_ERR_CUDA;
        ++i;
    }
    return queued != SFA_OK ? queued : joined;
}

// ------------------------------------------------------------------------------------
// Split-KV forward that allocates nothing.
//
// Some callers cannot hand this library a workspace: a process whose GPU memory is owned
// by an allocator it may not call into (a custom caching pool, a framework that forbids
// allocation while it is running), or code paths that must never call cudaMalloc or
// cudaFree because those synchronise the device.  For them the split-KV scratch lives in
// a fixed array of device memory inside this library, reserved once per GPU when the
// library's kernels are loaded there and kept until the process exits.
// ------------------------------------------------------------------------------------
namespace sfa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SFA_NOALLOC_SCRATCH_BYTES];

constexpr int NOALLOC_MAX_DEVICES = 256;
std::mutex g_noalloc_mutex;
struct NoallocCache {
    unsigned long long ctx_id;  // the context the address belongs to (0: none yet)
    void *ptr;
};
NoallocCache g_noalloc[NOALLOC_MAX_DEVICES] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (CUDA contexts get ids that are never
// reused within a process), or 0 if it cannot be read.
unsigned long long current_ctx_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device.  In host code the array's
// name only stands for it, so the address is looked up with the device current
// (cudaGetSymbolAddress) and cached per device together with the id of the context it
// was found in.  A device reset (cudaDeviceReset) replaces the primary context and may
// move the array; the next call then sees a new context id and looks the address up again.
sfa_status noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SFA_ERR_CUDA;
    if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return SFA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoallocCache &c = g_noalloc[dev];
    const unsigned long long ctx = current_ctx_id();  // 0 before the runtime has set a context current
    if (!c.ptr || ctx == 0 || c.ctx_id != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SFA_ERR_CUDA;
        c.ptr = p;
        c.ctx_id = current_ctx_id();  // the lookup has made the device's primary context current
    }
    *out = c.ptr;
    return SFA_OK;
}

}  // namespace
}  // namespace sfa

extern "C" sfa_status sfa_forward_split_noalloc(const sfa_attn_desc *d, const void *q, const void *k,
                                                const void *v, const int32_t *frames, const int32_t *counts,
                                                void *o, float *lse, int32_t n_split, int32_t *dev_status,
                                                sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (n_split < 1 || n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (n_split > 1 && split_ws_bytes(d, n_split) > (size_t)SFA_NOALLOC_SCRATCH_BYTES)
        return SFA_ERR_INVALID_ARG;  // needs more scratch than the fixed array holds
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, frames, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    if (n_split == 1)
        return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s)
                           : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s);
    void *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SFA_OK) return st;
    float *ws_lse = reinterpret_cast<float *>(static_cast<char *>(scratch) + split_ws_o_bytes(d, n_split));
    return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s, n_split, scratch, ws_lse)
                       : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s, n_split, scratch, ws_lse);
}

// ------------------------------------------------------------------------------------
// Two branches in one launch ("ISPA", §2.1 Dual-Stream Warmup): the local and the history
// key sets of the same queries run as one grid; the partials give the local branch and,
// merged by LSE, the full attention.
// ------------------------------------------------------------------------------------
extern "C" sfa_status sfa_forward_dual_workspace(const sfa_attn_desc *d, int32_t n_split, size_t *bytes)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (!bytes || n_split < 0 || 2 * n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (n_split == 0) {
        int k0, k1;
        auto_splits(d, 2, 0, k0, k1);
        *bytes = sched_ws_bytes(d, k0, k1);
        return SFA_OK;
    }
    *bytes = split_ws_bytes(d, 2 * n_split);
    return SFA_OK;
}

extern "C" sfa_status sfa_forward_dual(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                       const int32_t *frames_local, const int32_t *counts_local,
                                       const int32_t *frames_hist, const int32_t *counts_hist, void *o_local,
                                       float *lse_local, void *o_full, float *lse_full, int32_t n_split,
                                       void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                       sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (n_split < 0 || 2 * n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, frames_local, counts_local, o_full, lse_full);
    if (st != SFA_OK) return st;
    if (!frames_hist || !counts_hist || !o_local || !lse_local || reinterpret_cast<uintptr_t>(o_local) % 16)
        return SFA_ERR_INVALID_ARG;
    if (n_split == 0) {  // scheduled: the local branch one range per unit, the history branch split
        Schedule sc;
        auto_splits(d, 2, 0, sc.k0, sc.k1);
        const int slices = sc.k0 + sc.k1;
        if (!workspace || workspace_bytes < sched_ws_bytes(d, sc.k0, sc.k1) ||
            reinterpret_cast<uintptr_t>(workspace) % 256)
            return SFA_ERR_INVALID_ARG;
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        sc.items = reinterpret_cast<int2 *>(ws + split_ws_bytes(d, slices));
        float *ws_lse = reinterpret_cast<float *>(ws + split_ws_o_bytes(d, slices));
        cudaStream_t s = as_cuda(stream);
        return d->d == 128 ? launch<128>(d, q, k, v, frames_local, counts_local, o_full, lse_full, dev_status, s,
                                         sc.k0, workspace, ws_lse, nullptr, 0, 0, frames_hist, counts_hist, o_local,
                                         lse_local, &sc)
                           : launch<64>(d, q, k, v, frames_local, counts_local, o_full, lse_full, dev_status, s,
                                        sc.k0, workspace, ws_lse, nullptr, 0, 0, frames_hist, counts_hist, o_local,
                                        lse_local, &sc);
    }
    const size_t need = split_ws_bytes(d, 2 * n_split);
    if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256)
        return SFA_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    float *ws_lse = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + split_ws_o_bytes(d, 2 * n_split));
    return d->d == 128 ? launch<128>(d, q, k, v, frames_local, counts_local, o_full, lse_full, dev_status, s, n_split,
                                     workspace, ws_lse, nullptr, 0, 0, frames_hist, counts_hist, o_local, lse_local)
                       : launch<64>(d, q, k, v, frames_local, counts_local, o_full, lse_full, dev_status, s, n_split,
                                    workspace, ws_lse, nullptr, 0, 0, frames_hist, counts_hist, o_local, lse_local);
}

// ------------------------------------------------------------------------------------
// Key-block lists (hierarchical selection): each (b, h, t, query block of 256 rows) has
// its own sorted list of 128-token key blocks.
// ------------------------------------------------------------------------------------
extern "C" sfa_status sfa_forward_blocks_split_workspace(const sfa_attn_desc *d, int32_t n_split, size_t *bytes)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (!bytes || n_split < 0 || n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (n_split == 0) {
        int k0, k1;
        auto_splits(d, 1, (d->P + KEY_BLOCK - 1) / KEY_BLOCK, k0, k1);
        *bytes = sched_ws_bytes(d, k0, 0);
        return SFA_OK;
    }
    *bytes = n_split == 1 ? 0 : split_ws_bytes(d, n_split);
    return SFA_OK;
}

extern "C" sfa_status sfa_forward_blocks_split(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                               const int32_t *blocks, const int32_t *counts, void *o, float *lse,
                                               int32_t n_split, void *workspace, size_t workspace_bytes,
                                               int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if ((int64_t)d->T_kv * ((d->P + KEY_BLOCK - 1) / KEY_BLOCK) >= ((int64_t)1 << 31)) return SFA_ERR_INVALID_ARG;
    if (n_split < 0 || n_split > d->d / 8) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, blocks, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    const int nblk = (d->P + KEY_BLOCK - 1) / KEY_BLOCK;
    if (n_split == 0) {  // scheduled: ranges chosen here, longest first
        Schedule sc;
        auto_splits(d, 1, nblk, sc.k0, sc.k1);
        if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < sched_ws_bytes(d, sc.k0, 0))
            return SFA_ERR_INVALID_ARG;
        if (sc.k0 == 1)  // one range per unit: the plain launch
            return d->d == 128 ? launch<128>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr,
                                             nullptr, 0, nblk)
                               : launch<64>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr,
                                            nullptr, 0, nblk);
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        sc.items = reinterpret_cast<int2 *>(ws + (sc.k0 > 1 ? split_ws_bytes(d, sc.k0) : 0));
        void *ws_o = sc.k0 > 1 ? workspace : nullptr;
        float *ws_lse = sc.k0 > 1 ? reinterpret_cast<float *>(ws + split_ws_o_bytes(d, sc.k0)) : nullptr;
        return d->d == 128 ? launch<128>(d, q, k, v, blocks, counts, o, lse, dev_status, s, sc.k0, ws_o, ws_lse,
                                         nullptr, 0, nblk, nullptr, nullptr, nullptr, nullptr, &sc)
                           : launch<64>(d, q, k, v, blocks, counts, o, lse, dev_status, s, sc.k0, ws_o, ws_lse, nullptr,
                                        0, nblk, nullptr, nullptr, nullptr, nullptr, &sc);
    }
    if (n_split == 1)
        return d->d == 128 ? launch<128>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr, nullptr,
                                         0, nblk)
                           : launch<64>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr, nullptr,
                                        0, nblk);
    const size_t need = split_ws_bytes(d, n_split);
    if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256)
        return SFA_ERR_INVALID_ARG;
    float *ws_lse = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + split_ws_o_bytes(d, n_split));
    return d->d == 128 ? launch<128>(d, q, k, v, blocks, counts, o, lse, dev_status, s, n_split, workspace, ws_lse,
                                     nullptr, 0, nblk)
                       : launch<64>(d, q, k, v, blocks, counts, o, lse, dev_status, s, n_split, workspace, ws_lse,
                                    nullptr, 0, nblk);
}

extern "C" sfa_status sfa_forward_blocks(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                         const int32_t *blocks, const int32_t *counts, void *o, float *lse,
                                         int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if ((int64_t)d->T_kv * ((d->P + KEY_BLOCK - 1) / KEY_BLOCK) >= ((int64_t)1 << 31)) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    st = check_buffers(d, q, k, v, blocks, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    const int nblk = (d->P + KEY_BLOCK - 1) / KEY_BLOCK;
    return d->d == 128 ? launch<128>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr, nullptr, 0,
                                     nblk)
                       : launch<64>(d, q, k, v, blocks, counts, o, lse, dev_status, s, 1, nullptr, nullptr, nullptr, 0,
                                    nblk);
}

// ------------------------------------------------------------------------------------
// Paged key/value caches: a per-head table maps each logical key/value frame to the
// physical frame slot that holds it, so per-head caches of different contents need no
// compaction.
// ------------------------------------------------------------------------------------
extern "C" sfa_status sfa_forward_paged(const sfa_attn_desc *d, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *slots, int32_t n_slots,
                                        const int32_t *frames, const int32_t *counts, void *o, float *lse,
                                        int32_t *dev_status, sfa_stream_t stream)
{
    sfa_status st = check_desc(d);
    if (st != SFA_OK) return st;
    if (n_slots < 1 || (int64_t)n_slots * d->P >= ((int64_t)1 << 31)) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!slots) return SFA_ERR_INVALID_ARG;
    st = check_buffers(d, q, k_cache, v_cache, frames, counts, o, lse);
    if (st != SFA_OK) return st;
    cudaStream_t s = as_cuda(stream);
    return d->d == 128 ? launch<128>(d, q, k_cache, v_cache, frames, counts, o, lse, dev_status, s, 1, nullptr,
                                     nullptr, slots, n_slots)
                       : launch<64>(d, q, k_cache, v_cache, frames, counts, o, lse, dev_status, s, 1, nullptr,
                                    nullptr, slots, n_slots);
}
