// Frame-sparse softmax attention forward for sm_100a (B200).
//
// What it computes ("LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de
// Video Largo", §2 Mecanismo Central and §Complejidad): every query frame t attends only
// to the key/value tokens of the frames in A(h, t), so a query costs O(|A| P d) instead
// of O(T P d).  Per row it also emits the log-sum-exp of its scaled scores, the state
// that "ISPA" (§2.1, Atención Descomponible) uses to merge partial attentions.
//
// How, on one SM per work unit (b, h, t, 128-row query tile):
//   * the frame list of (h, t) is walked as runs of consecutive frames; each run is one
//     contiguous token interval, cut into 128-key tiles, so unattended frames are never
//     loaded and only the last tile of a run is partial;
//   * warp 4 (one thread) streams Q once and K/V tiles through a 3-stage (d = 128) or
//     4-stage (d = 64) shared-memory ring with TMA, 128-byte swizzled;
//   * warp 5 (one thread) issues tcgen05.mma: S = Q K^T into one of two TMEM S buffers
//     while the softmax works on the other, then O += P V with P read from TMEM;
//     a partial last tile uses an MMA N (for S) and K (for P V) rounded up to 16 only;
//   * warps 0-3 (one thread per query row = TMEM lane) run the online softmax in fp32
//     (exp2 with the scale folded into one FMA; O is rescaled only when a row's running
//     max grows by more than 2^8, otherwise the stale max is kept), write P as bf16 into
//     TMEM, and finally normalise O, stage it in shared memory and TMA-store it, clipped
//     to the frame, plus the fp32 LSE.
// Every mbarrier wait is bounded; a wait that runs out records SFA_ERR_TIMEOUT, the CTA
// drains its in-flight copies and MMAs, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

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
constexpr int NUM_THREADS = 192;        // warps 0-3 softmax, 4 TMA producer, 5 MMA issuer
constexpr int PRODUCER_WARP = 4;
constexpr int MMA_WARP = 5;
constexpr float RESCALE_LOG2 = 8.0f;    // keep a stale row max while the new one is < 2^8 above
constexpr uint32_t DEFAULT_TIMEOUT_US = 2000000;  // 2 s; a healthy wait lasts microseconds
constexpr uint32_t DRAIN_TIMEOUT_US = 2000000;
constexpr uint32_t MAX_SPINS = 1u << 30;           // backstop should the timer not advance

// tensor-memory columns (512 allocated: 2 x S fp32, O fp32, 2 x P bf16)
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P0 = 384, TM_P1 = 448, TM_COLS = 512;

template <int D>
struct Cfg {
    static constexpr int KBOX = D / 64;                 // 128-byte swizzle boxes per row
    static constexpr int BOX_BYTES = 128 * 128;         // 128 rows x 64 bf16
    static constexpr int TILE_BYTES = BM * D * 2;       // one Q / K / V / O tile
    static constexpr int NS = D == 128 ? 3 : 4;         // K/V ring depth
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_K = TILE_BYTES;
    static constexpr int SMEM_V = SMEM_K + NS * TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_V + NS * TILE_BYTES;
    static constexpr int SMEM_BYTES = SMEM_BAR + 256 + 1024;  // + barriers, + alignment slack
};

struct FwdArgs {
    int32_t B, H, Tq, T_kv, P, Amax;
    int32_t n_qtiles;
    float scale_log2;  // softmax scale * log2(e)
    const int32_t *frames;
    const int32_t *counts;
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
// Number of K/V tiles for a frame list, or -1 if the list is not strictly increasing
// inside [0, T_kv).
__device__ int count_tiles(const int32_t *fl, int cnt, int T_kv, int P)
{
    int tiles = 0, a = 0, prev = -1;
    while (a < cnt) {
        const int f0 = __ldg(fl + a);
        if (f0 <= prev || f0 >= T_kv) return -1;
        int f1 = f0;
        ++a;
        while (a < cnt && __ldg(fl + a) == f1 + 1) {
            ++f1;
            ++a;
        }
        if (f1 >= T_kv) return -1;
        prev = f1;
        tiles += ((f1 - f0 + 1) * P + BN - 1) / BN;
    }
    return tiles;
}

// Walks the attended tokens as runs of consecutive frames, 128 keys at a time.
struct KvIter {
    const int32_t *fl;
    int n, a, P, pos, end;
    __device__ void init(const int32_t *f, int cnt, int P_)
    {
        fl = f;
        n = cnt;
        a = 0;
        P = P_;
        pos = 0;
        end = 0;
    }
    __device__ void next(int &start, int &nvalid)
    {
        if (pos >= end) {
            const int f0 = __ldg(fl + a);
            int f1 = f0;
            ++a;
            while (a < n && __ldg(fl + a) == f1 + 1) {
                ++f1;
                ++a;
            }
            pos = f0 * P;
            end = (f1 + 1) * P;
        }
        start = pos;
        nvalid = min(BN, end - pos);
        pos += BN;
    }
};

__device__ __forceinline__ uint32_t mma_n(int nvalid) { return (uint32_t)((nvalid + 15) & ~15); }

// ----------------------------------------------------------------- roles
template <int D>
__device__ void producer_role(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                              const FwdArgs &a, uint32_t sbase, int b, int h, int t, int qt, const int32_t *fl,
                              int cnt, int n_tiles, const Ctl &ctl)
{
    using C = Cfg<D>;
    const uint32_t bars = sbase + C::SMEM_BAR;
    const uint32_t q_full = bars + 8 * (3 * C::NS);
    if (n_tiles <= 0) return;
    mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
#pragma unroll
    for (int kb = 0; kb < C::KBOX; ++kb)
        tma_load_5d(sbase + C::SMEM_Q + kb * C::BOX_BYTES, tm_q, q_full, kb * 64, qt * BM, t, h, b);

    // K/V of one (h, t) are re-read by every query tile of the frame: keep them in L2
    const uint64_t policy = l2_policy_evict_last();
    KvIter it;
    it.init(fl, cnt, a.P);
    int j = 0;
    for (; j < n_tiles; ++j) {
        const int s = j % C::NS;
        const uint32_t k_full = bars + 8 * s, v_full = bars + 8 * (C::NS + s);
        const uint32_t kv_empty = bars + 8 * (2 * C::NS + s);
        if (j >= C::NS && !wait_bar(kv_empty, ((j / C::NS) - 1) & 1, ctl)) break;
        int start, nv;
        it.next(start, nv);
        mbar_arrive_expect_tx(k_full, C::TILE_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KBOX; ++kb)
            tma_load_4d(sbase + C::SMEM_K + s * C::TILE_BYTES + kb * C::BOX_BYTES, tm_k, k_full, kb * 64, start,
                        h, b, policy);
        mbar_arrive_expect_tx(v_full, C::TILE_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KBOX; ++kb)
            tma_load_4d(sbase + C::SMEM_V + s * C::TILE_BYTES + kb * C::BOX_BYTES, tm_v, v_full, kb * 64, start,
                        h, b, policy);
    }
    if (*ctl.abort) {  // let the copies still in flight land before the CTA exits
        wait_drain(q_full, 0);
        for (int jj = (j > C::NS ? j - C::NS : 0); jj < j; ++jj) {
            const int s = jj % C::NS;
            wait_drain(bars + 8 * s, (jj / C::NS) & 1);
            wait_drain(bars + 8 * (C::NS + s), (jj / C::NS) & 1);
        }
    }
}

template <int D>
__device__ __forceinline__ void issue_s(uint32_t t_s, uint32_t s_q, uint32_t s_k, uint32_t n)
{
    // S[128 x n] = Q[128 x D] K[n x D]^T, both K-major; one MMA per 16 elements of D.
    const uint32_t idesc = idesc_bf16_f32(BM, n, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * Cfg<D>::BOX_BYTES + (kk & 3) * 32;
        mma_ss(t_s, sdesc_sw128(s_q + off, 16, 1024), sdesc_sw128(s_k + off, 16, 1024), idesc, kk > 0);
    }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t t_o, uint32_t t_p, uint32_t s_v, uint32_t n, bool accumulate)
{
    // O[128 x D] += P[128 x n] V[n x D]; P (bf16, 2 per column) from TMEM, V MN-major
    // (D contiguous): 8-key groups 1024 B apart, 64-wide D blocks one box apart.
    const uint32_t idesc = idesc_bf16_f32(BM, D, true);
    for (uint32_t kk = 0; kk < n / 16; ++kk)
        mma_ts(t_o, t_p + kk * 8, sdesc_sw128(s_v + kk * 2048, Cfg<D>::BOX_BYTES, 1024), idesc,
               (accumulate || kk > 0) ? 1u : 0u);
}

template <int D>
__device__ void mma_role(const FwdArgs &a, uint32_t sbase, uint32_t tmem, const int32_t *fl, int cnt,
                         int n_tiles, const Ctl &ctl)
{
    using C = Cfg<D>;
    const uint32_t bars = sbase + C::SMEM_BAR;
    const uint32_t q_full = bars + 8 * (3 * C::NS);
    const uint32_t s_full0 = q_full + 8, p_full0 = q_full + 24, o_done = q_full + 40, drain = q_full + 48;
    const uint32_t o_final = q_full + 56;
    const uint32_t s_q = sbase + C::SMEM_Q;
    if (n_tiles <= 0) return;
    bool issued = false;
    KvIter it;
    it.init(fl, cnt, a.P);
    int st, nv_cur, nv_next = 0;
    it.next(st, nv_cur);
    if (wait_bar(q_full, 0, ctl) && wait_bar(bars, 0, ctl)) {
        tc_fence_after();
        issue_s<D>(tmem + TM_S0, s_q, sbase + C::SMEM_K, mma_n(nv_cur));
        tc_commit(s_full0);
        issued = true;
        for (int j = 0; j < n_tiles; ++j) {
            if (j + 1 < n_tiles) {  // S for the next tile overlaps the softmax of this one
                it.next(st, nv_next);
                const int s1 = (j + 1) % C::NS;
                if (!wait_bar(bars + 8 * s1, ((j + 1) / C::NS) & 1, ctl)) break;
                tc_fence_after();
                issue_s<D>(tmem + ((j + 1) & 1 ? TM_S1 : TM_S0), s_q, sbase + C::SMEM_K + s1 * C::TILE_BYTES,
                           mma_n(nv_next));
                tc_commit(s_full0 + 8 * ((j + 1) & 1));
            }
            const int s = j % C::NS;
            if (!wait_bar(p_full0 + 8 * (j & 1), (j >> 1) & 1, ctl)) break;
            if (!wait_bar(bars + 8 * (C::NS + s), (j / C::NS) & 1, ctl)) break;
            tc_fence_after();
            issue_pv<D>(tmem + TM_O, tmem + ((j & 1) ? TM_P1 : TM_P0), sbase + C::SMEM_V + s * C::TILE_BYTES,
                        mma_n(nv_cur), j > 0);
            tc_commit(bars + 8 * (2 * C::NS + s));  // K/V stage free
            tc_commit(o_done);                      // O holds tiles 0..j
            nv_cur = nv_next;
            // single-phase signal for the epilogue: with parity waits alone, the P V of the
            // last two tiles can both be pending and would be indistinguishable
            if (j == n_tiles - 1) tc_commit(o_final);
        }
    }
    if (*ctl.abort && issued) {  // wait for the tensor cores before TMEM is released
        tc_commit(drain);
        wait_drain(drain, 0);
    }
}

template <int D>
__device__ void softmax_role(const CUtensorMap *tm_o, const FwdArgs &a, uint8_t *smem, uint32_t sbase,
                             uint32_t tmem, int b, int h, int t, int qt, const int32_t *fl, int cnt, int n_tiles,
                             bool bad_set, const Ctl &ctl)
{
    using C = Cfg<D>;
    const uint32_t bars = sbase + C::SMEM_BAR;
    const uint32_t q_full = bars + 8 * (3 * C::NS);
    const uint32_t s_full0 = q_full + 8, p_full0 = q_full + 24, o_done = q_full + 40;
    const uint32_t o_final = q_full + 56;
    volatile int32_t *epi_ok = reinterpret_cast<volatile int32_t *>(smem + C::SMEM_BAR + 224);
    const int row = threadIdx.x;  // query row inside the tile == TMEM lane
    const int warp = row >> 5;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = a.scale_log2;

    float m_used = -INFINITY;  // running row max (log2 units, scale folded in)
    float l = 0.f;             // running row sum of exp2(s*sl2 - m_used)
    bool alive = true;
    KvIter it;
    it.init(fl, cnt, a.P);
    for (int j = 0; j < n_tiles; ++j) {
        int st, nv;
        it.next(st, nv);
        const bool got = wait_bar(s_full0 + 8 * (j & 1), (j >> 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, got)) {
            alive = false;
            break;
        }
        tc_fence_after();
        const uint32_t t_s = lane_base + ((j & 1) ? TM_S1 : TM_S0);
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (c * 32 < nv) tmem_ld32(t_s + c * 32, sr[c]);
        tmem_wait_ld();

        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c * 32 < nv) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (nv < BN && c * 32 + i >= nv) sr[c][i] = __float_as_uint(-INFINITY);
                    mx = fmaxf(mx, __uint_as_float(sr[c][i]));
                }
            }
        }
        const float m_cand = mx * sl2;
        const bool resc = m_cand > m_used + RESCALE_LOG2;
        const float m_new = resc ? m_cand : m_used;
        const float alpha = ex2_approx(m_used - m_new);  // 0 on the first tile, 1 if unchanged
        const float neg_m = -m_new;

        // P = exp2(s * scale * log2e - m) as bf16 pairs, stored to TMEM chunk by chunk
        const uint32_t t_p = lane_base + ((j & 1) ? TM_P1 : TM_P0);
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c * 32 < nv) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c][2 * i]), sl2, neg_m));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c][2 * i + 1]), sl2, neg_m));
                    rs0 += p0;
                    rs1 += p1;
                    pk[i] = pack_bf16x2(p0, p1);
                }
                tmem_st16(t_p + c * 16, pk);
            }
        }

        // O must be rescaled before P V of this tile accumulates into it; the warp
        // does it together (tcgen05.ld/st are warp-wide) after P V of tile j-1 is done.
        // The parity wait is unambiguous here: S of tile j was committed after P V of
        // tile j-2, so only P V of tile j-1 can still be pending.
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
            const bool done = wait_bar(o_done, (j - 1) & 1, ctl);
            if (!__all_sync(0xffffffffu, done)) {
                alive = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_base + TM_O + c * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tmem_st32(lane_base + TM_O + c * 32, o);
            }
        }
        l = l * alpha + (rs0 + rs1);
        m_used = m_new;

        tmem_wait_st();
        tc_fence_before();
        if (!((a.debug_flags & SFA_DEBUG_STALL_SOFTMAX) && j == 0)) mbar_arrive(p_full0 + 8 * (j & 1));
    }

    // ---- epilogue: O / l -> bf16 -> swizzled smem (the Q tile's space) -> TMA store
    bool have = alive;
    if (have && n_tiles > 0) {
        const bool done = wait_bar(o_final, 0, ctl);
        have = __all_sync(0xffffffffu, done);
    }
    if ((row & 31) == 0) epi_ok[warp] = have ? 1 : 0;
    named_bar_sync(1, BM);
    const bool write = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
    if (write) {
        const float inv_l = n_tiles > 0 ? 1.f / l : 0.f;
        uint8_t *s_o = smem + C::SMEM_Q;
        if (n_tiles > 0) tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            if (n_tiles > 0) {
                tmem_ld32(lane_base + TM_O + c * 32, o);
                tmem_wait_ld();
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
    named_bar_sync(1, BM);
    if (write && row == 0) {
#pragma unroll
        for (int kb = 0; kb < C::KBOX; ++kb)
            tma_store_5d(tm_o, sbase + C::SMEM_Q + kb * C::BOX_BYTES, kb * 64, qt * BM, t, h, b);
        tma_store_commit();
        tma_store_wait_read_all();
    }
    const int p = qt * BM + row;
    if (write && p < a.P) {
        float lse;
        if (bad_set) lse = __int_as_float(0x7fc00000);  // NaN marks a rejected frame list
        else if (n_tiles == 0) lse = -INFINITY;
        else lse = (m_used + log2f(l)) * 0.69314718055994530942f;
        a.lse[((int64_t)(b * a.H + h) * a.Tq + t) * a.P + p] = lse;
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

    // work unit: (b, h, t, query tile), query tile fastest so that the tiles sharing
    // one frame's K/V run side by side
    int x = blockIdx.x;
    const int qt = x % a.n_qtiles;
    x /= a.n_qtiles;
    const int t = x % a.Tq;
    x /= a.Tq;
    const int h = x % a.H;
    const int b = x / a.H;
    const int32_t *fl = a.frames + ((int64_t)h * a.Tq + t) * a.Amax;
    const int cnt = __ldg(a.counts + h * a.Tq + t);
    int n_tiles = (cnt >= 0 && cnt <= a.Amax) ? count_tiles(fl, cnt, a.T_kv, a.P) : -1;
    const bool bad_set = n_tiles < 0;
    if (bad_set) n_tiles = 0;
    volatile int32_t *skip = reinterpret_cast<volatile int32_t *>(smem + C::SMEM_BAR + 248);

    if (threadIdx.x == 0) {
        for (int i = 0; i < 3 * C::NS; ++i) mbar_init(bars + 8 * i, 1);  // K full, V full, K/V empty
        const uint32_t q_full = bars + 8 * (3 * C::NS);
        mbar_init(q_full, 1);
        mbar_init(q_full + 8, 1);        // S full x2 (tcgen05.commit)
        mbar_init(q_full + 16, 1);
        mbar_init(q_full + 24, BM);      // P full x2 (every softmax thread)
        mbar_init(q_full + 32, BM);
        mbar_init(q_full + 40, 1);       // O done (P V committed)
        mbar_init(q_full + 48, 1);       // drain
        mbar_init(q_full + 56, 1);       // O final (after the last P V)
        *abort_flag = 0;
        // once a CTA has timed out, the ones that start later skip their work
        *skip = (a.status && *reinterpret_cast<volatile int32_t *>(a.status) == SFA_ERR_TIMEOUT) ? 1 : 0;
        fence_mbar_init();
        if (bad_set) report(a.status, SFA_ERR_BAD_SET);
    }
    if (warp == PRODUCER_WARP && lane == 0) {
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

    if (warp == PRODUCER_WARP) {
        if (lane == 0) producer_role<D>(&tm_q, &tm_k, &tm_v, a, sbase, b, h, t, qt, fl, cnt, n_tiles, ctl);
    } else if (warp == MMA_WARP) {
        if (lane == 0) mma_role<D>(a, sbase, tmem, fl, cnt, n_tiles, ctl);
        __syncwarp();
    } else {
        if (!skipped) softmax_role<D>(&tm_o, a, smem, sbase, tmem, b, h, t, qt, fl, cnt, n_tiles, bad_set, ctl);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
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

template <int D>
sfa_status launch(const sfa_attn_desc *d, const void *q, const void *k, const void *v, const int32_t *frames,
                  const int32_t *counts, void *o, float *lse, int32_t *dev_status, cudaStream_t stream)
{
    using C = Cfg<D>;
    CUtensorMap tq, tk, tv, to;
    const uint64_t P = d->P, Tq = d->Tq, Lkv = (uint64_t)d->T_kv * d->P;
    {
        const uint64_t dims[5] = {(uint64_t)D, P, Tq, (uint64_t)d->H, (uint64_t)d->B};
        const uint64_t st[4] = {(uint64_t)d->q_stride[2] * 2, P * d->q_stride[2] * 2, (uint64_t)d->q_stride[1] * 2,
                                (uint64_t)d->q_stride[0] * 2};
        if (!encode(&tq, q, 5, dims, st)) return SFA_ERR_UNSUPPORTED;
        const uint64_t so[4] = {(uint64_t)d->o_stride[2] * 2, P * d->o_stride[2] * 2, (uint64_t)d->o_stride[1] * 2,
                                (uint64_t)d->o_stride[0] * 2};
        if (!encode(&to, o, 5, dims, so)) return SFA_ERR_UNSUPPORTED;
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
    a.lse = lse;
    a.status = dev_status;
    a.timeout_ns = (uint64_t)(d->timeout_us ? d->timeout_us : DEFAULT_TIMEOUT_US) * 1000;
    a.debug_flags = d->debug_flags;

    const int64_t grid = (int64_t)d->B * d->H * d->Tq * a.n_qtiles;
    if (cudaFuncSetAttribute(sfa_forward_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
        return SFA_ERR_CUDA;
    sfa_forward_kernel<D><<<(unsigned)grid, NUM_THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, a);
    return launch_status();
}

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_forward(const sfa_attn_desc *d, const void *q, const void *k, const void *v,
                                  const int32_t *frames, const int32_t *counts, void *o, float *lse,
                                  int32_t *dev_status, sfa_stream_t stream)
{
    if (!d) return SFA_ERR_INVALID_ARG;
    if (d->B < 0 || d->H < 1 || d->Tq < 1 || d->T_kv < 1 || d->P < 1 || d->Amax < 1) return SFA_ERR_INVALID_ARG;
    if (d->d != 64 && d->d != 128) return SFA_ERR_UNSUPPORTED;
    if (!(d->scale > 0.f) || !std::isfinite(d->scale)) return SFA_ERR_INVALID_ARG;
    if ((int64_t)d->Tq * d->P >= ((int64_t)1 << 31) || (int64_t)d->T_kv * d->P >= ((int64_t)1 << 31))
        return SFA_ERR_INVALID_ARG;
    const int64_t grid = (int64_t)d->B * d->H * d->Tq * ((d->P + BM - 1) / BM);
    if (grid >= ((int64_t)1 << 31)) return SFA_ERR_INVALID_ARG;
    if (d->B == 0) return SFA_OK;
    if (!q || !k || !v || !o || !lse || !frames || !counts) return SFA_ERR_INVALID_ARG;
    for (const void *p : {q, k, v, (const void *)o})
        if (reinterpret_cast<uintptr_t>(p) % 16) return SFA_ERR_INVALID_ARG;
    if (!stride_ok(d->q_stride, d->d) || !stride_ok(d->k_stride, d->d) || !stride_ok(d->v_stride, d->d) ||
        !stride_ok(d->o_stride, d->d))
        return SFA_ERR_INVALID_ARG;
    cudaStream_t s = as_cuda(stream);
    return d->d == 128 ? launch<128>(d, q, k, v, frames, counts, o, lse, dev_status, s)
                       : launch<64>(d, q, k, v, frames, counts, o, lse, dev_status, s);
}
