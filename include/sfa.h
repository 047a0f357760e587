/*
 * sfa.h - frame-sparse attention for video diffusion transformers on B200 (sm_100a).
 *
 * C ABI of libsfa.so.  Three operations, all asynchronous on the caller's CUDA
 * stream, all on device buffers that the caller owns:
 *
 *   sfa_build_sets  attended frame sets A(h, t), one sorted list per (head, query frame)
 *   sfa_forward     softmax attention of every query frame over the tokens of A(h, t)
 *                   only, writing O (bf16) and the per-row log-sum-exp (fp32)
 *   sfa_lse_merge   merge of two partial attentions (e.g. local + history branch)
 *
 * plus variants of the forward (host buffers, paged caches, split-KV, two branches in one
 * launch), the hierarchical block selection of Light Forcing (sfa_hsa_select +
 * sfa_forward_blocks) and ARL2's inter-frame gated-delta branch (sfa_gdn_forward).
 *
 * Conventions
 *   - A video has T latent frames of P tokens each; token i belongs to frame i / P.
 *     Query frame t (0 <= t < Tq) sits at frame t + q_off of the key/value timeline
 *     (0 <= frame < T_kv).  Frame lists hold absolute key/value frame indices.
 *   - Device pointers are plain CUDA device addresses (cudaMalloc / torch memory).
 *     The library never allocates device memory and keeps no state between calls,
 *     apart from per-process caches of the CUDA driver entry points it uses (to
 *     encode TMA descriptors and to read the current context's id) and what
 *     sfa_forward_split_noalloc needs: a fixed scratch array of device memory on
 *     every GPU that loads the library, whose contents persist from one call to the
 *     next, and its cached device address.
 *   - Every call validates its arguments on the host first and returns a status;
 *     nothing is printed and nothing throws across the ABI.  Launch errors come
 *     back as SFA_ERR_CUDA.  Errors that only the GPU can see (a malformed frame
 *     list, a wait that ran out) are written to an optional device status word.
 *   - sfa_stream_t is a cudaStream_t (0 = legacy default stream).
 */
#ifndef SFA_H_
#define SFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sfa_stream_t; /* same type as cudaStream_t */

typedef enum {
    SFA_OK = 0,
    SFA_ERR_INVALID_ARG = 1,  /* a size, pointer, stride or parameter is out of range   */
    SFA_ERR_UNSUPPORTED = 2,  /* valid, but outside what this build implements (e.g. d) */
    SFA_ERR_CUDA = 3,         /* a CUDA runtime / driver call or kernel launch failed   */
    SFA_ERR_TIMEOUT = 4,      /* device: a pipeline wait hit its time limit             */
    SFA_ERR_BAD_SET = 5       /* device: a frame list is unsorted, repeated or out of range,
                                 or a count is outside [0, Amax]                        */
} sfa_status;

/* Human-readable name of a status code (static storage, never NULL). */
const char *sfa_error_string(sfa_status s);

/* Library version as 10000*major + 100*minor + patch. */
int32_t sfa_version(void);

/* ------------------------------------------------------------------------------------
 * Attended frame sets
 * ------------------------------------------------------------------------------------
 * Kinds, for query frame t at timeline frame c = t + q_off:
 *
 *   SFA_SET_DENSE     A = {0 .. T_kv-1}: full attention (the set LVSA replaces;
 *                     "LVSA: Atención Dispersa Libre de Entrenamiento para Difusión de
 *                     Video Largo", §2 Mecanismo Central).
 *   SFA_SET_LVSA      A = G_s ∪ W(c) (same page, §2.1 and §2.2):
 *                       G_s  = { f : f mod T_per == step mod T_per }, rotating global
 *                              anchors, each frame an anchor once per T_per steps;
 *                       W(c) = window of W frames centred on c (an even W puts the extra
 *                              frame after c), shifted inside [0, T_kv), then grown one
 *                              frame at a time, alternating after/before c (after first,
 *                              a side at the end of the video hands its turn over), until
 *                              |A| = min(C, T_kv).  The window never shrinks: if G_s ∪ W
 *                              already exceeds C, A is larger than C.
 *   SFA_SET_LOCAL     A = current chunk ∪ the n_prev frames before it, where the chunk of
 *                     c is [c0, c0 + chunk_len), c0 = c - c mod chunk_len ("Head Forcing",
 *                     §2: local heads keep the current block and its nearest frames).
 *   SFA_SET_ANCHOR    A = {0 .. n_sink-1} ∪ LOCAL (same page: anchor heads add the first
 *                     latent frames; "ISPA", §2.1: local branch = current + sink).
 *   SFA_SET_MEMORY    A = ANCHOR ∪ extra[h] (same page: memory heads add selected
 *                     history frames; the selection itself is the caller's).
 *   SFA_SET_EXPLICIT  A = extra[h] (any caller-chosen list, e.g. a history branch).
 *
 * Every list is clipped to [0, T_kv), sorted ascending and free of repeats.
 */
typedef enum {
    SFA_SET_DENSE = 0,
    SFA_SET_LVSA = 1,
    SFA_SET_LOCAL = 2,
    SFA_SET_ANCHOR = 3,
    SFA_SET_MEMORY = 4,
    SFA_SET_EXPLICIT = 5
} sfa_set_kind;

#define SFA_MAX_HEADS 1024

typedef struct {
    int32_t T_kv;      /* key/value frames, >= 1                                       */
    int32_t Tq;        /* query frames, >= 1, with q_off + Tq <= T_kv                   */
    int32_t q_off;     /* timeline frame of query frame 0, >= 0                          */
    int32_t C;         /* LVSA budget, >= 1                                              */
    int32_t W;         /* LVSA base window, >= 1                                         */
    int32_t T_per;     /* LVSA anchor period, >= 1                                       */
    int32_t step;      /* LVSA denoising step s, >= 0                                    */
    int32_t n_sink;    /* ANCHOR/MEMORY: leading sink frames, >= 0                      */
    int32_t n_prev;    /* LOCAL/ANCHOR/MEMORY: frames kept before the chunk, >= 0        */
    int32_t chunk_len; /* LOCAL/ANCHOR/MEMORY: frames per chunk, >= 1                    */
} sfa_set_params;

/*
 * Upper bound on |A(h, t)| over all heads and query frames for these parameters:
 * the smallest Amax that sfa_build_sets accepts.  head_kind: host array [H].
 * Returns SFA_ERR_INVALID_ARG for bad parameters or kinds.
 */
sfa_status sfa_set_max_count(const sfa_set_params *p, int32_t H, const int32_t *head_kind,
                             int32_t n_extra, int32_t *amax_out);

/*
 * Build A(h, t) for every head h < H and query frame t < Tq.
 *   p          host pointer to the parameters above.
 *   head_kind  host array [H] of sfa_set_kind, 1 <= H <= SFA_MAX_HEADS.
 *   extra      device int32 [H][n_extra], entries outside [0, T_kv) ignored (use -1 as
 *              padding); may be NULL when n_extra == 0.  Read by MEMORY/EXPLICIT heads.
 *   frames     device int32 [H][Tq][Amax], written: the sorted list, then -1 padding.
 *   counts     device int32 [H][Tq], written: |A(h, t)|.
 *   Amax       must be >= sfa_set_max_count(...), else SFA_ERR_INVALID_ARG.
 * One thread per (h, t); output is bit-identical whatever the launch.
 */
sfa_status sfa_build_sets(const sfa_set_params *p, int32_t H, const int32_t *head_kind,
                          const int32_t *extra, int32_t n_extra, int32_t *frames,
                          int32_t *counts, int32_t Amax, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Frame-sparse attention forward
 * ------------------------------------------------------------------------------------
 * For each batch b, head h and query row i of query frame t = i / P, with the key set
 *   K(h, t) = ∪_{f in A(h,t)} [f*P, (f+1)*P):
 *     s_j = scale * q_i . k_j,  O_i = sum_j softmax(s)_j v_j,  LSE_i = ln sum_j exp(s_j)
 * ("LVSA", §2 Mecanismo Central: attention restricted to A(t); §Complejidad: cost
 *  O(|A(t)| P d) per query; "ISPA", §2.1: the per-row LSE kept by the kernel is what
 *  makes two partial attentions mergeable).  An empty set gives O_i = 0, LSE_i = -inf.
 * Attention is bidirectional inside every attended frame; nothing is token-causal.
 *
 * Layout: q [B][H][Tq*P][d], k and v [B][H][T_kv*P][d], o like q, all bf16, addressed
 * as base + b*stride[0] + h*stride[1] + token*stride[2] + e (strides in elements; the
 * d elements of a token are contiguous).  BHLD and BLHD layouts both fit.  Base
 * addresses must be 16-byte aligned and strides multiples of 8 elements (TMA rule).
 * lse is fp32 [B][H][Tq*P], contiguous.
 * frames / counts as written by sfa_build_sets ([H][Tq][Amax], [H][Tq]; shared by all
 * batch entries); each list must be strictly increasing inside [0, T_kv).
 * Supported: d in {64, 128}, any P >= 1, any scale > 0 (the usual is 1/sqrt(d)).
 * dev_status: optional device int32 (may be NULL), which the caller sets to 0; a
 * device-side error stores its sfa_status there (first error wins) and the affected
 * query tile's outputs are then unspecified.
 * timeout_us: time limit of every pipeline wait inside the kernel (0 = 2 s).  When a wait
 * runs out, its CTA stores SFA_ERR_TIMEOUT, drains its copies and tensor-core work, frees
 * its tensor memory and exits; CTAs that start after that see the status and skip their
 * work, so a broken pipeline costs about one time limit, not one per CTA.
 */
typedef struct {
    int32_t B, H, Tq, T_kv, P, d;
    float scale;
    int32_t Amax;
    int64_t q_stride[3]; /* batch, head, token */
    int64_t k_stride[3];
    int64_t v_stride[3];
    int64_t o_stride[3];
    uint32_t timeout_us;   /* limit of every pipeline wait in the kernel, microseconds;
                              0 = 2 s (a healthy wait lasts microseconds) */
    uint32_t debug_flags;  /* SFA_DEBUG_* below; 0 in normal use */
} sfa_attn_desc;

/* Test hook: the softmax warps never publish their first probability tile, so the
 * tensor-core warp's wait for it runs out; the call must then report SFA_ERR_TIMEOUT
 * through dev_status and still return cleanly. */
#define SFA_DEBUG_STALL_SOFTMAX 1u

sfa_status sfa_forward(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                       const int32_t *frames, const int32_t *counts, void *o, float *lse,
                       int32_t *dev_status, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Host buffers in and out
 * ------------------------------------------------------------------------------------
 * sfa_forward ("LVSA", §2 Mecanismo Central: attention of every query frame over A(t)
 * only) for Q, K, V in host memory, with O and LSE written back to host memory, the
 * copies and the attention run as one pipeline on the device: the (batch, head-group)
 * chunks go in order, and the copy of chunk i+1 to the device, the attention of chunk i
 * (two streams in turn, so that one kernel's last wave overlaps the next one's first)
 * and the copy of chunk i-1 back overlap.
 *   q_host, k_host, v_host  bf16 [B][H][Tq*P][d] and [B][H][T_kv*P][d], contiguous (the
 *                      descriptor's strides are not used); page-locked (cudaHostAlloc /
 *                      pinned torch memory) for the copies to overlap, else the copies
 *                      run synchronously and the result is the same.
 *   frames, counts     device lists as for sfa_forward.
 *   o_host             bf16 [B][H][Tq*P][d], lse_host fp32 [B][H][Tq*P], host, written.
 *   n_chunks           chunks per call (>= 1): min(H, n_chunks / B) head groups per batch
 *                      entry (at least one).
 *   workspace          caller-owned device memory of sfa_forward_host_workspace bytes,
 *                      256-byte aligned: the device copies of Q, K, V, O and LSE.
 * The call creates its own streams and events and destroys them before it returns (work
 * queued on them completes normally); all its work is ordered after the work already on
 * `stream`, and `stream` waits for all of it, like a single kernel: synchronise `stream`
 * before reading o_host / lse_host.  On an error the work already queued still joins
 * `stream`.  Argument errors are returned before anything is queued.
 */
sfa_status sfa_forward_host_workspace(const sfa_attn_desc *desc, size_t *bytes);

sfa_status sfa_forward_host(const sfa_attn_desc *desc, const void *q_host, const void *k_host, const void *v_host,
                            const int32_t *frames, const int32_t *counts, void *o_host, float *lse_host,
                            int32_t n_chunks, void *workspace, size_t workspace_bytes, int32_t *dev_status,
                            sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Paged key/value caches
 * ------------------------------------------------------------------------------------
 * ("Head Forcing", §2: every head keeps its own cache — local, anchor or memory — of
 *  different frames.)  sfa_forward with the keys and values read through a per-head slot
 * table: logical key/value frame f of head h lives in physical frame slot
 * slots[h * T_kv + f] of k_cache / v_cache, so caches are updated by rewriting slots and
 * the table, never by compacting tensors.
 *   k_cache, v_cache  bf16 [B][H][n_slots * P][d] with desc->k_stride / v_stride.
 *   slots             device int32 [H][T_kv] (shared by the batch); only entries of
 *                     frames that appear in a list are read, each must lie in
 *                     [0, n_slots) (else SFA_ERR_BAD_SET through dev_status).
 *   desc->T_kv        logical frames (the range of the frame lists), n_slots >= 1.
 * List entries whose slots are consecutive are read as one contiguous run.  Every slot
 * may hold arbitrary data: rows past a run's end are never used.
 */
sfa_status sfa_forward_paged(const sfa_attn_desc *desc, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *slots, int32_t n_slots, const int32_t *frames, const int32_t *counts,
                             void *o, float *lse, int32_t *dev_status, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Split-KV forward (same result as sfa_forward, for short or uneven grids)
 * ------------------------------------------------------------------------------------
 * The key tiles of every (batch, head, query frame, 128-row query tile) are cut into
 * n_split contiguous ranges that run as separate CTAs; each writes a partial O and LSE
 * into the workspace, and the partials are merged by their LSE ("ISPA", §2.1: the LSE
 * state makes partial attentions over disjoint key sets mergeable; the merge is
 * sfa_lse_merge's rule over n_split branches).  Use it when B*H*Tq*ceil(P/128) is small
 * next to the number of SMs or the sets differ a lot in size between heads.
 *
 * n_split = 0 (scheduled): the library chooses the number of ranges (Amax taken as every
 * unit's length, the launch modelled as waves of equal pieces plus the merge); with one
 * range per unit (many full waves) the call is sfa_forward's launch.  With several, a
 * one-CTA kernel first counts every list's key tiles on the device and orders the CTAs
 * longest range first, so that the block scheduler runs a longest-first schedule.  The result is
 * the same attention; the order of the partial merge is fixed by the ranges, so a call
 * is deterministic.  sfa_forward_split_plan reports the choice.
 *
 * sfa_forward_split_workspace: bytes of device workspace for this descriptor and
 *   n_split (0 when n_split == 1).  0 <= n_split <= d/8, else SFA_ERR_INVALID_ARG.
 * sfa_forward_split: arguments as sfa_forward, plus n_split and a caller-owned device
 *   workspace of at least that many bytes, 256-byte aligned (unused when n_split == 1;
 *   its contents are scratch and are overwritten).  Partial O is rounded to bf16 before
 *   the merge, in fp32, rounds it once more.
 */
sfa_status sfa_forward_split_workspace(const sfa_attn_desc *desc, int32_t n_split, size_t *bytes);

/* The key-tile ranges per unit a scheduled call (n_split = 0) uses for this descriptor:
 * n_lists = 1 for sfa_forward_split (key_blocks = 0) or sfa_forward_blocks_split
 * (key_blocks = 1), 2 for sfa_forward_dual (k_first for the local lists, k_second for
 * the history lists).  k_second may be NULL. */
sfa_status sfa_forward_split_plan(const sfa_attn_desc *desc, int32_t n_lists, int32_t key_blocks, int32_t *k_first,
                                  int32_t *k_second);

sfa_status sfa_forward_split(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                             const int32_t *frames, const int32_t *counts, void *o, float *lse,
                             int32_t n_split, void *workspace, size_t workspace_bytes, int32_t *dev_status,
                             sfa_stream_t stream);

/*
 * sfa_forward_split_noalloc: sfa_forward_split for callers that cannot allocate device
 * memory for the library (their memory belongs to an allocator they may not call into,
 * or they must not call cudaMalloc / cudaFree, which synchronise the device).  The pages
 * have no counterpart: this is an interface convenience, not part of the method.
 *   - The workspace is a fixed array of SFA_NOALLOC_SCRATCH_BYTES inside the library,
 *     reserved on every GPU where the library's kernels are loaded and held until the
 *     process exits.  The call allocates nothing (no cudaMalloc, no cudaFree, no
 *     allocating library routine); the caller still passes inputs and outputs.
 *   - The first call on a device looks up the array's device address with that device
 *     current (cudaGetSymbolAddress) and caches it with the id of the current context;
 *     make that first call before any stream capture on the device.  After a device
 *     reset (cudaDeviceReset) the context id changes and the next call looks the
 *     address up again, so that call too should come before any stream capture.
 *   - Requests needing more than SFA_NOALLOC_SCRATCH_BYTES of workspace (see
 *     sfa_forward_split_workspace) return SFA_ERR_INVALID_ARG without launching.
 *     n_split == 1 needs no workspace.
 *   - Every call shares the one array, which keeps the previous call's contents (nothing
 *     in it has to start at zero: each call writes every partial it reads).  Calls
 *     that can overlap on the GPU (different streams, or different host threads on the
 *     same device) race on it: serialise them.
 */
#define SFA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

sfa_status sfa_forward_split_noalloc(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                                     const int32_t *frames, const int32_t *counts, void *o, float *lse,
                                     int32_t n_split, int32_t *dev_status, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Two branches in one launch
 * ------------------------------------------------------------------------------------
 * ("ISPA", §2.1 Dual-Stream Warmup: the local branch — current frame and sink — and the
 *  full attention are both needed; with disjoint local and history key sets the full
 *  attention is the LSE merge of the two branches.)  One grid runs the local lists and
 * the history lists of the same queries (each cut into n_split key-tile ranges as in
 * sfa_forward_split); one merge pass then writes
 *   o_local, lse_local = attention over the local lists, and
 *   o_full,  lse_full  = the LSE merge of both branches (attention over the union when
 *                        the two lists of a (h, t) are disjoint).
 * frames_local / counts_local and frames_hist / counts_hist: [H][Tq][Amax] / [H][Tq] as
 * sfa_build_sets writes them (the same Amax).  o_local and o_full use desc->o_stride.
 * sfa_forward_dual_workspace: bytes of workspace for n_split (1 <= 2 n_split <= d/8).
 * n_split = 0 schedules the launch as sfa_forward_split does: the local lists keep one
 * key-tile range per unit, the history lists get the number of ranges the library
 * chooses (sfa_forward_split_plan with n_lists = 2), and the CTAs run longest range first.
 * The workspace must be 256-byte aligned; partial O is rounded to bf16 before the merge.
 */
sfa_status sfa_forward_dual_workspace(const sfa_attn_desc *desc, int32_t n_split, size_t *bytes);

sfa_status sfa_forward_dual(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                            const int32_t *frames_local, const int32_t *counts_local,
                            const int32_t *frames_hist, const int32_t *counts_hist, void *o_local,
                            float *lse_local, void *o_full, float *lse_full, int32_t n_split,
                            void *workspace, size_t workspace_bytes, int32_t *dev_status,
                            sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Hierarchical sparse attention (HSA): selection of key blocks, and attention over them
 * ------------------------------------------------------------------------------------
 * ("Resumen Técnico: LIGHT FORCING", §2.2 Atención Dispersa Jerárquica: query and key
 *  tokens are mean-pooled per block and per frame; each query block picks a few history
 *  frames with the frame-level pooled keys, then the critical blocks inside them with the
 *  block-level pooled keys; attention runs over the picked frame-block pairs only.)
 *
 * Blocks.  A key block is 128 consecutive tokens of one frame: block b of frame f holds
 * tokens [f*P + 128 b, f*P + min(128 (b+1), P)) and has id f * nblk + b, with
 * nblk = ceil(P / 128).  A query block is 256 consecutive query rows of one frame (the
 * last one of a frame holds the rest): nqb = ceil(P / 256) per frame.
 *
 * Selection, per (b, h, query frame t, query block), with c = t + q_off and the chunk
 * [c0, c0 + chunk_len), c0 = c - c mod chunk_len:
 *   always  = every block of the frames {0 .. n_sink-1} ∪ [c0 - n_prev, c0 + chunk_len)
 *             (the sink and the local window; clipped to [0, T_kv));
 *   history = the other frames before c0;
 *   score   = (mean of the block's query rows) . (mean of the frame's or block's keys),
 *             in fp32;
 *   frames  = the k_frames history frames of highest score; then
 *   picked  = the k_blocks blocks of highest score among all blocks of those frames
 *             (equal scores: the smaller id first; k larger than the candidates keeps
 *             them all);
 *   list    = always ∪ picked, sorted ascending.
 *
 * sfa_hsa_max_count: the list length bound for these parameters,
 *   (n_sink + n_prev + chunk_len) * nblk + min(k_blocks, k_frames * nblk): the smallest
 *   Amax that sfa_hsa_select accepts.
 * sfa_hsa_workspace: bytes of device workspace sfa_hsa_select needs (the pooled keys
 *   and queries, fp32).
 * sfa_hsa_select: writes the lists.
 *   desc      B, H, Tq, T_kv, P, d, q_stride, k_stride as for sfa_forward; desc->Amax =
 *             list capacity (>= sfa_hsa_max_count); scale, v/o strides unused.
 *   p         q_off, n_sink, n_prev, chunk_len used (p->T_kv, p->Tq must equal the
 *             descriptor's); the LVSA fields are ignored.
 *   q, k      bf16, laid out as for sfa_forward.
 *   workspace caller-owned device memory, >= sfa_hsa_workspace bytes, 256-byte aligned;
 *             scratch, overwritten.
 *   blocks    device int32 [B][H][Tq][nqb][Amax], written: the sorted list, -1 padding.
 *   counts    device int32 [B][H][Tq][nqb], written: list lengths.
 *   k_frames >= 0, k_blocks >= 0; T_kv * nblk <= 65536.
 * sfa_forward_blocks: sfa_forward over key-block lists: query rows of query block i of
 *   frame t attend to the tokens of the blocks in blocks[b][h][t][i] (layout and Amax as
 *   sfa_hsa_select writes them; each list strictly increasing inside [0, T_kv * nblk),
 *   else SFA_ERR_BAD_SET through dev_status).  Other arguments as sfa_forward.
 */
sfa_status sfa_hsa_max_count(const sfa_set_params *p, int32_t P, int32_t k_frames, int32_t k_blocks,
                             int32_t *amax_out);

sfa_status sfa_hsa_workspace(const sfa_attn_desc *desc, size_t *bytes);

sfa_status sfa_hsa_select(const sfa_attn_desc *desc, const sfa_set_params *p, int32_t k_frames,
                          int32_t k_blocks, const void *q, const void *k, void *workspace,
                          size_t workspace_bytes, int32_t *blocks, int32_t *counts, sfa_stream_t stream);

/* Selection with the pooled keys kept from an earlier call.  The history frames of an
 * autoregressive cache do not change while later chunks attend them, so their frame and
 * block means ("LIGHT FORCING", §2.2: token compression of the keys) need computing once:
 * sfa_hsa_pool_keys writes them into the workspace (the part sfa_hsa_select also fills),
 * and sfa_hsa_select_pooled pools the queries only and selects from the keys' means
 * already there.  sfa_hsa_pool_keys followed by sfa_hsa_select_pooled gives the lists
 * sfa_hsa_select gives for the same q and k, bit for bit.  Arguments as sfa_hsa_select;
 * the workspace must be the one the keys were pooled into, for the same descriptor
 * (B, H, T_kv, P, d); its other parts are overwritten. */
sfa_status sfa_hsa_pool_keys(const sfa_attn_desc *desc, const void *k, void *workspace, size_t workspace_bytes,
                             sfa_stream_t stream);

sfa_status sfa_hsa_select_pooled(const sfa_attn_desc *desc, const sfa_set_params *p, int32_t k_frames,
                                 int32_t k_blocks, const void *q, void *workspace, size_t workspace_bytes,
                                 int32_t *blocks, int32_t *counts, sfa_stream_t stream);

sfa_status sfa_forward_blocks(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                              const int32_t *blocks, const int32_t *counts, void *o, float *lse,
                              int32_t *dev_status, sfa_stream_t stream);

/* sfa_forward_blocks with the key tiles of every unit cut into n_split ranges and merged
 * by LSE, as sfa_forward_split does for frame lists; n_split = 0 schedules the launch
 * (the library's choice of ranges, longest first).  Workspace: the size
 * sfa_forward_blocks_split_workspace gives for the same descriptor and n_split. */
sfa_status sfa_forward_blocks_split_workspace(const sfa_attn_desc *desc, int32_t n_split, size_t *bytes);

sfa_status sfa_forward_blocks_split(const sfa_attn_desc *desc, const void *q, const void *k, const void *v,
                                    const int32_t *blocks, const int32_t *counts, void *o, float *lse,
                                    int32_t n_split, void *workspace, size_t workspace_bytes,
                                    int32_t *dev_status, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * ARL2 inter-frame branch: gated delta rule over frames
 * ------------------------------------------------------------------------------------
 * ("Resumen Técnico: Asistir Localmente, Recordar Linealmente (ARL2)", §2.1 Rama
 *  Inter-Cuadro and §2.2 Gestión del Estado de Memoria.)  Per (batch b, head h) a state
 * S [d][d] (fp32) replaces the KV cache.  For frames N = 0 .. T-1 in order:
 *     O_N = Q'_N S_{N-1}                       (every token of the frame reads the same,
 *                                              pre-update state: frame-level access)
 *     S_N = alpha_N S_{N-1} + K'_N^T diag(beta_N) (V'_N - K'_N S_{N-1})   if update != 0
 *     S_N = S_{N-1}                                                        if update == 0
 * (update == 0 is the read-only access of the intermediate denoising steps).
 *   q, k, v, o  bf16 [B][H][T*P][d] with the strides in the descriptor (d contiguous; 16-byte
 *               aligned bases, strides multiples of 8 elements); q, k, v are the
 *               feature-mapped projections Q', K', V'.
 *   alpha       fp32 [B][H][T] (one forget factor per frame), contiguous.
 *   beta        fp32 [B][H][T*P] (one step size per token, >= 0), contiguous.  A negative
 *               or NaN beta is reported as SFA_ERR_INVALID_ARG in dev_status and its
 *               token is left out of the update.
 *   state_in    fp32 [B][H][d][d] (row = key dimension), contiguous, or NULL for zeros.
 *   state_out   fp32 [B][H][d][d]; may be the same buffer as state_in.
 * Method: the update is linear in the state, S_N = alpha_N S_{N-1} - M_N S_{N-1} + B_N
 * with M_N = K'^T diag(beta) K' and B_N = K'^T diag(beta) V' of frame N alone.  A first
 * kernel forms M_N and B_N of every frame at once on the tensor cores; a second runs the
 * recurrence (one d x d x d product per frame) in several CTAs per (batch, head), each of
 * which also computes O for its share of the frame's tokens.  The tensor cores read M_N,
 * S and sqrt(beta)-scaled K', V' as bf16; M_N S accumulates, B_N and the state are kept
 * in fp32.  The result does not depend on the launch shape.  Supported: d = 128, any
 * P >= 1, any T >= 1.
 * workspace: update != 0 needs a device workspace of sfa_gdn_workspace bytes (256-byte
 *   aligned; scratch, overwritten; M_N and B_N of every frame), else SFA_ERR_INVALID_ARG.
 *   With update == 0 it is not used and may be NULL.
 */
typedef struct {
    int32_t B, H, T, P, d;
    int64_t q_stride[3]; /* batch, head, token (elements) */
    int64_t k_stride[3];
    int64_t v_stride[3];
    int64_t o_stride[3];
    uint32_t timeout_us;  /* limit of every wait inside the kernel; 0 = 2 s */
    uint32_t debug_flags; /* SFA_DEBUG_* below; 0 in normal use */
} sfa_gdn_desc;

/* Test hook: the element-wise warps of the recurrence kernel never signal the input state
 * ready, so its tensor-core warp's first wait runs out; the call must then report
 * SFA_ERR_TIMEOUT through dev_status, its copies in flight must land, and it must return
 * cleanly. */
#define SFA_DEBUG_STALL_GDN_STATE 2u

sfa_status sfa_gdn_workspace(const sfa_gdn_desc *desc, size_t *bytes);

sfa_status sfa_gdn_forward(const sfa_gdn_desc *desc, const void *q, const void *k, const void *v,
                           const float *alpha, const float *beta, const float *state_in, float *state_out,
                           void *o, int32_t update, void *workspace, size_t workspace_bytes,
                           int32_t *dev_status, sfa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * LSE merge
 * ------------------------------------------------------------------------------------
 * ("ISPA", §2.1 Dual-Stream Warmup and contribution 2: local and history branches of
 *  attention, fused after the fact through their log-sum-exp.)  Per row r, with
 *  M = max(L1, L2):
 *     L = M + ln(exp(L1 - M) + exp(L2 - M)),  O = exp(L1 - L) O1 + exp(L2 - L) O2.
 * A branch with L = -inf contributes nothing; both -inf gives O = 0, L = -inf.
 * If the two branches cover disjoint key sets, (O, L) is attention over their union.
 *   o1, o2, o: device bf16 [rows][d], contiguous rows; lse1, lse2, lse: device fp32
 *   [rows].  o / lse may alias o1 / lse1 (in-place).  d in {64, 128}; rows >= 0.
 * Math in fp32; O rounded to bf16 once.
 */
sfa_status sfa_lse_merge(int64_t rows, int32_t d, const void *o1, const float *lse1,
                         const void *o2, const float *lse2, void *o, float *lse,
                         sfa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SFA_H_ */
