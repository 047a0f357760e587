// Attended-frame-set builder: one thread per (head, query frame).
//
// LVSA ("LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de Video Largo",
// §2 Mecanismo Central): A(t) = G_s ∪ W(t).  G_s are the frames whose index is
// congruent to s mod T_per (rotating global anchors, §2.1); W(t) is a window of W
// frames around t, shifted inside the video and grown over anchor overlaps until the
// set holds min(C, T) frames (§2.2).  Per-head cache kinds ("Head Forcing", §2; "ISPA",
// §2.1) are unions of a chunk-aligned local block, leading sink frames and a
// caller-given list.  The output is a sorted list padded with -1 and its length.
#include <cstdint>

#include "sfa.h"
#include "sfa_internal.h"

namespace sfa {
namespace {

struct SetArgs {
    int32_t T, Tq, q_off, C, W, T_per, step, n_sink, n_prev, chunk_len;
    int32_t H, n_extra, Amax;
    const int32_t *extra;
    int32_t *frames;
    int32_t *counts;
    int8_t kind[SFA_MAX_HEADS];
};

__device__ bool in_extra(const int32_t *ex, int32_t n, int32_t f)
{
    for (int32_t e = 0; e < n; ++e)
        if (ex[e] == f) return true;
    return false;
}

__global__ void __launch_bounds__(128) build_sets_kernel(const __grid_constant__ SetArgs a)
{
    const int32_t idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= a.H * a.Tq) return;
    const int32_t h = idx / a.Tq;
    const int32_t t = idx - h * a.Tq;
    const int32_t T = a.T;
    const int32_t c = t + a.q_off;
    const int kind = a.kind[h];
    int32_t *out = a.frames + (int64_t)idx * a.Amax;
    int32_t n = 0;

    if (kind == SFA_SET_LVSA) {
        const int32_t phase = a.step % a.T_per;
        int32_t lo, hi;
        if (a.W >= T) {
            lo = 0;
            hi = T - 1;
        } else {
            lo = c - (a.W - 1) / 2;
            hi = lo + a.W - 1;
            if (lo < 0) {
                lo = 0;
                hi = a.W - 1;
            } else if (hi > T - 1) {
                hi = T - 1;
                lo = T - a.W;
            }
        }
        // |G_s ∪ [lo, hi]| = |G_s| + frames of the window that are not anchors
        int32_t size = phase < T ? (T - 1 - phase) / a.T_per + 1 : 0;
        for (int32_t f = lo; f <= hi; ++f) size += (f % a.T_per != phase);
        const int32_t target = a.C < T ? a.C : T;
        bool future_turn = true;
        while (size < target && !(lo == 0 && hi == T - 1)) {
            const bool grow_future = (future_turn && hi < T - 1) || lo == 0;
            const int32_t f = grow_future ? ++hi : --lo;
            size += (f % a.T_per != phase);
            future_turn = !future_turn;
        }
        for (int32_t f = 0; f < T && n < a.Amax; ++f)
            if (f % a.T_per == phase || (f >= lo && f <= hi)) out[n++] = f;
    } else if (kind == SFA_SET_DENSE) {
        for (int32_t f = 0; f < T && n < a.Amax; ++f) out[n++] = f;
    } else {
        const int32_t c0 = c - c % a.chunk_len;
        const int32_t lo = c0 - a.n_prev;
        const int32_t hi = c0 + a.chunk_len - 1;
        const int32_t *ex = a.extra ? a.extra + (int64_t)h * a.n_extra : nullptr;
        const bool local = kind != SFA_SET_EXPLICIT;
        const bool sink = kind == SFA_SET_ANCHOR || kind == SFA_SET_MEMORY;
        const bool listed = (kind == SFA_SET_MEMORY || kind == SFA_SET_EXPLICIT) && ex;
        for (int32_t f = 0; f < T && n < a.Amax; ++f) {
            const bool m = (local && f >= lo && f <= hi) || (sink && f < a.n_sink) ||
                           (listed && in_extra(ex, a.n_extra, f));
            if (m) out[n++] = f;
        }
    }
    a.counts[idx] = n;
    for (int32_t i = n; i < a.Amax; ++i) out[i] = -1;
}

sfa_status check_params(const sfa_set_params *p, int32_t H, const int32_t *head_kind, int32_t n_extra)
{
    if (!p || !head_kind || H < 1 || H > SFA_MAX_HEADS || n_extra < 0) return SFA_ERR_INVALID_ARG;
    if (p->T_kv < 1 || p->Tq < 1 || p->q_off < 0 || (int64_t)p->q_off + p->Tq > p->T_kv)
        return SFA_ERR_INVALID_ARG;
    for (int32_t h = 0; h < H; ++h) {
        const int32_t k = head_kind[h];
        if (k < SFA_SET_DENSE || k > SFA_SET_EXPLICIT) return SFA_ERR_INVALID_ARG;
        if (k == SFA_SET_LVSA && (p->C < 1 || p->W < 1 || p->T_per < 1 || p->step < 0))
            return SFA_ERR_INVALID_ARG;
        if ((k == SFA_SET_LOCAL || k == SFA_SET_ANCHOR || k == SFA_SET_MEMORY) &&
            (p->chunk_len < 1 || p->n_prev < 0 || p->n_sink < 0))
            return SFA_ERR_INVALID_ARG;
    }
    return SFA_OK;
}

int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

}  // namespace
}  // namespace sfa

using namespace sfa;

extern "C" sfa_status sfa_set_max_count(const sfa_set_params *p, int32_t H, const int32_t *head_kind,
                                        int32_t n_extra, int32_t *amax_out)
{
    if (!amax_out) return SFA_ERR_INVALID_ARG;
    const sfa_status st = check_params(p, H, head_kind, n_extra);
    if (st != SFA_OK) return st;
    const int64_t T = p->T_kv;
    int64_t best = 0;
    for (int32_t h = 0; h < H; ++h) {
        int64_t b = 0;
        switch (head_kind[h]) {
        case SFA_SET_DENSE: b = T; break;
        case SFA_SET_LVSA: {
            const int64_t phase = p->step % p->T_per;
            const int64_t anchors = phase < T ? (T - 1 - phase) / p->T_per + 1 : 0;
            b = max64(min64(p->C, T), min64(T, anchors + p->W));
            break;
        }
        case SFA_SET_LOCAL: b = min64(T, (int64_t)p->chunk_len + p->n_prev); break;
        case SFA_SET_ANCHOR: b = min64(T, (int64_t)p->chunk_len + p->n_prev + p->n_sink); break;
        case SFA_SET_MEMORY: b = min64(T, (int64_t)p->chunk_len + p->n_prev + p->n_sink + n_extra); break;
        case SFA_SET_EXPLICIT: b = min64(T, n_extra); break;
        }
        best = max64(best, b);
    }
    *amax_out = (int32_t)best;
    return SFA_OK;
}

extern "C" sfa_status sfa_build_sets(const sfa_set_params *p, int32_t H, const int32_t *head_kind,
                                     const int32_t *extra, int32_t n_extra, int32_t *frames,
                                     int32_t *counts, int32_t Amax, sfa_stream_t stream)
{
    int32_t bound = 0;
    const sfa_status st = sfa_set_max_count(p, H, head_kind, n_extra, &bound);
    if (st != SFA_OK) return st;
    if (!frames || !counts || Amax < 1 || Amax < bound) return SFA_ERR_INVALID_ARG;
    if (n_extra > 0 && !extra) return SFA_ERR_INVALID_ARG;
    if ((int64_t)H * p->Tq * Amax > (int64_t)1 << 31) return SFA_ERR_INVALID_ARG;

    SetArgs a;
    a.T = p->T_kv;
    a.Tq = p->Tq;
    a.q_off = p->q_off;
    a.C = p->C;
    a.W = p->W;
    a.T_per = p->T_per > 0 ? p->T_per : 1;
    a.step = p->step;
    a.n_sink = p->n_sink;
    a.n_prev = p->n_prev;
    a.chunk_len = p->chunk_len > 0 ? p->chunk_len : 1;
    a.H = H;
    a.n_extra = n_extra;
    a.Amax = Amax;
    a.extra = n_extra > 0 ? extra : nullptr;
    a.frames = frames;
    a.counts = counts;
    for (int32_t h = 0; h < SFA_MAX_HEADS; ++h) a.kind[h] = h < H ? (int8_t)head_kind[h] : 0;

    const int32_t n = H * p->Tq;
    const int32_t threads = 128;
    build_sets_kernel<<<(n + threads - 1) / threads, threads, 0, as_cuda(stream)>>>(a);
    return launch_status();
}
