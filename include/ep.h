/*
 * ep.h -- C ABI of the B200 (sm_100a) MoE expert-parallel dispatch/combine
 * library (libep.so).
 *
 * The operation is DeepEP's: route every token to the experts of its top-k
 * choice and bring the expert outputs back (all-to-all dispatch and
 * combine for MoE, with FP8 dispatch -- chinainews.com, "DeepSeek releases
 * DeepEP", feature list; Wallstreetcn/lbkrs review, feature list;
 * dataforcee.us rewrite, "Technological Views and Benefits": tokens travel
 * to their experts and the results are merged back).  Here the
 * expert-parallel ranks are logical partitions of one GPU's memory: rank r
 * owns the G = E / R consecutive experts [r*G, (r+1)*G), and "sending to
 * rank r" means writing into rank r's segment of one expert-contiguous
 * receive buffer.
 *
 * Notation: T tokens, hidden size H, top-k slots per token, E experts,
 * R ranks.  idx[T,k] expert ids (-1 = dropped slot), w[T,k] fp32 gate
 * weights, x[T,H] bf16 hidden states.  N = T*k is the receive capacity.
 * All arrays are dense row-major in device memory unless stated otherwise.
 *
 * Conventions for every entry point:
 *  - Asynchronous: work is enqueued on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) and the call returns without waiting.
 *  - Stateless: nothing is kept between calls, so calls on different
 *    streams with different buffers may run concurrently.  (Two
 *    exceptions, both described below: ep_get_layout_noalloc shares one
 *    scratch array per device between its calls, and the testing switch
 *    ep_debug_expire_first_wait is process-wide.)
 *  - The caller allocates and owns every buffer; the library allocates no
 *    device memory.
 *  - Argument errors are returned before anything is enqueued; nothing is
 *    written then.  EP_ERR_CUDA means a launch failed; the message is in
 *    ep_last_error_string().  Nothing ever traps on the device: problems
 *    found on the device are written to the caller's optional error word
 *    d_err (device int32, may be NULL; never cleared by the library) --
 *    EP_ERR_INDEX for a bad expert id (its slot is treated as dropped),
 *    EP_ERR_TIMEOUT if a kernel's bounded wait for its own asynchronous
 *    copies gave up (it then stops early instead of hanging).
 *  - Pointers must be 16-byte aligned unless stated otherwise.
 *  - Kernels are launched with programmatic stream serialization: one may
 *    be scheduled as the previous kernel on `stream` finishes, and it waits
 *    for that kernel (griddepcontrol.wait) before reading anything.  Only
 *    the one-token-per-CTA kernel of ep_layout_dispatch releases its
 *    successor early, once its CTAs have only their final stores left; the
 *    successor must still wait before reading.  A caller's kernel launched
 *    after one of these with the same attribute must wait the same way
 *    before reading their output; one launched without it sees plain
 *    stream order.
 */
#ifndef EP_H_
#define EP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int ep_status_t;

#define EP_OK 0
#define EP_ERR_INVALID_ARG 1 /* null/misaligned pointer, bad size        */
#define EP_ERR_UNSUPPORTED 2 /* valid request outside the built limits   */
#define EP_ERR_CUDA 3        /* a CUDA call failed; see ep_last_error_string */
#define EP_ERR_INDEX 4       /* device-side: an expert id outside [-1, E) */
#define EP_ERR_TIMEOUT 5     /* device-side: a bounded wait for an async copy
                                gave up; that call's output is incomplete */

#define EP_MAX_K 32    /* top-k slots per token            */
#define EP_MAX_E 1024  /* experts                          */
#define EP_MAX_R 64    /* logical ranks                    */

/* Version of this ABI (incremented on any signature change, and when the
 * workspace a call needs changes): 5. */
int ep_abi_version(void);

/* Message of the last error returned on this host thread ("" if none). */
const char *ep_last_error_string(void);

/* Number of kernels this library has launched in this process. */
uint64_t ep_kernel_launches(void);

/*
 * Bytes of device workspace ep_get_layout needs for (T, k, E, R); 0 when the
 * single-CTA or cluster kernel applies (then ws may be NULL).  The kernel
 * depends on the slots T*k: up to 2048 one CTA; below 65536 one cluster of
 * up to 16 CTAs; from 65536 to 2^19 one CTA on each SM (a cooperative
 * launch; workspace: 16 bytes of barrier counters plus (E + R) * 161 int32
 * counts), unless that workspace would exceed 256 KiB, when the cluster
 * again; above 2^19 the tiled pair (16 bytes plus one row of E + R counts
 * per tile).  A launch refused for co-residency (for instance fewer free
 * SMs than CTAs in a green context) falls back to the cluster kernel.
 */
size_t ep_layout_workspace_bytes(int T, int k, int E, int R);

/*
 * ep_get_layout -- the dispatch layout: who goes where.
 *
 * The pages describe per-rank senders that each push a token to every
 * peer rank that needs it (frogred8 blog, "Implementation of SMs dedicated
 * to network communication": warp roles per peer, up to 8 NVLink peers),
 * which presumes per-rank counts, a token-in-rank mask and the prefix
 * offsets computed here; the layout follows the group-limited gating of
 * DeepSeek-V3 that DeepEP targets (chinainews.com item, paragraph on the
 * V3 paper).  Definitions (the pages give none; this is the reading):
 *   cnt_e[E]     number of slots (t,j) with idx[t,j] == e
 *   off_e[E+1]   exclusive prefix sum of cnt_e; off_e[E] = kept slots
 *   slot_pos[T,k] receive row of slot (t,j): off_e[e] + number of slots
 *                before (t,j) in token-major order with the same expert
 *                (stable: rows of one expert are in ascending token order);
 *                -1 for dropped slots
 *   recv_src[N]  token whose copy lands in each row; -1 past off_e[E]
 *   in_rank[T,R] (uint8) 1 iff token t has a kept slot in rank r's experts
 *   cnt_r[R]     tokens per rank (sum over t of in_rank[t,r])
 *   off_r[R+1]   exclusive prefix sum of cnt_r
 * Rank r's rows are [off_e[r*G], off_e[(r+1)*G]).
 *
 * idx          [T,k] int64 (idx_is_int64 != 0) or int32 expert ids; -1 drops
 *              a slot.  8-byte (int64) or 4-byte (int32) aligned.
 * T >= 0, 1 <= k <= min(E, EP_MAX_K), 1 <= E <= EP_MAX_E,
 * 1 <= R <= EP_MAX_R, E % R == 0, T*k < 2^31.
 * Outputs: int32 arrays 4-byte aligned, in_rank 1-byte aligned.
 * ws, ws_bytes  device scratch of at least ep_layout_workspace_bytes()
 *              bytes, 16-byte aligned.  It must be zero-filled before its
 *              first use; every call leaves its counters (the first 16
 *              bytes) at zero again and overwrites the rest, so one
 *              buffer serves a sequence of stream-ordered calls (not
 *              concurrent ones).
 * d_err        optional (may be NULL) device int32; set to EP_ERR_INDEX when
 *              an id outside [-1, E) is met (that slot is then dropped).
 *              Never cleared by the library.
 * Returns EP_OK, EP_ERR_INVALID_ARG, EP_ERR_UNSUPPORTED or EP_ERR_CUDA.
 */
ep_status_t ep_get_layout(const void *idx, int idx_is_int64, int T, int k,
                          int E, int R, int32_t *cnt_e, int32_t *cnt_r,
                          uint8_t *in_rank, int32_t *off_e, int32_t *off_r,
                          int32_t *slot_pos, int32_t *recv_src, void *ws,
                          size_t ws_bytes, int32_t *d_err, void *stream);

/*
 * ep_dispatch -- send each token to its experts' receive rows.
 *
 * DeepEP's dispatch (chinainews.com item, feature list: all-to-all for
 * MoE, FP8 support; Wallstreetcn/lbkrs review, feature list: FP8 dispatch;
 * frogred8 blog, TMA bulk copies and read-only non-coherent loads).  For
 * every slot (t,j) with slot_pos[t,j] = p >= 0:
 *   fp8 == 0:  recv[p, :] = x[t, :]                    (bf16 rows)
 *   fp8 != 0:  per 128-channel block b of token t,
 *              a = max |x[t, 128b : 128b+128]| (NaN propagates),
 *              a = max(a, 1e-4); s = a / 448 (fp32, round to nearest);
 *              recv[p, c] = e4m3(x[t, c] / s)  (fp32 quotient rounded to
 *              nearest; e4m3 round-to-nearest-even, saturating to +-448;
 *              NaN -> 0x7f);  recv_scale[p, b] = s.
 * x           [T,H] bf16.
 * slot_pos    [T,k] int32 from ep_get_layout (or ep_pad_layout); values
 *             outside [0, recv_rows) are skipped.
 * recv        [recv_rows, H] bf16 (fp8 == 0) or e4m3 bytes (fp8 != 0).  Rows
 *             no slot points at are left untouched.
 * recv_scale  [recv_rows, H/128] fp32 (fp8 != 0, 4-byte aligned), else
 *             ignored.
 * recv_rows   rows of recv (and recv_scale); slot rows outside
 *             [0, recv_rows) are skipped.  0 means T*k, the size of the
 *             packed layout; an aligned layout (ep_pad_layout) needs
 *             ep_aligned_rows(T, k, E, align).
 * T >= 0, 1 <= k <= EP_MAX_K, H > 0 with H % 8 == 0 (H % 128 == 0 for
 * fp8), T*k < 2^31.
 * num_sms     SMs to spread the work over.  0 = all of them: one CTA (or
 *             warp) per work item, waves of CTAs following one another as
 *             SMs free up.  n > 0: a persistent grid of the CTAs that n SMs
 *             hold at once, so that kernels on other streams keep the
 *             other SMs (the CTAs are not pinned to particular SMs).
 * d_err       optional device error word (see the conventions above).
 */
ep_status_t ep_dispatch(const void *x, int T, int H, int k,
                        const int32_t *slot_pos, int fp8, void *recv,
                        float *recv_scale, int recv_rows, int num_sms,
                        int32_t *d_err, void *stream);

/*
 * ep_layout_dispatch -- ep_get_layout followed by ep_dispatch, with the
 * same arguments and bit-identical outputs, in one kernel launch when the
 * batch is small.
 *
 * DeepEP serves small decode batches with separate low-latency kernels
 * (dataforcee.us rewrite, "Technological Views and Benefits": 128 tokens,
 * eight experts); on one GPU their cost is launch and dependency latency.
 * When T*k <= 8192, E * ceil(T/32) * 4 <= 32 KiB and H <= 16384 (for FP8
 * also H % 512 == 0 and a 16-byte aligned recv_scale), one kernel does it
 * all: every CTA works out, from all the ids, the layout entries of the
 * tokens it dispatches (one token per CTA when T + 1 CTAs fit on the GPU
 * at once), with no CTA waiting on another; otherwise the call enqueues
 * the two kernels of ep_get_layout and ep_dispatch (ep_kernel_launches
 * tells which ran).
 *
 * idx .. recv_src, ws, ws_bytes: as ep_get_layout (ws is needed only when
 * ep_layout_workspace_bytes(T, k, E, R) > 0, i.e. for T*k >= 65536).
 * x, H, fp8, recv, recv_scale, num_sms: as ep_dispatch.
 * d_err receives EP_ERR_INDEX for a bad id and EP_ERR_TIMEOUT as in
 * ep_dispatch.  All argument checks of both calls apply, before anything
 * is enqueued.
 */
ep_status_t ep_layout_dispatch(const void *idx, int idx_is_int64, int T,
                               int k, int E, int R, const void *x, int H,
                               int fp8, int32_t *cnt_e, int32_t *cnt_r,
                               uint8_t *in_rank, int32_t *off_e,
                               int32_t *off_r, int32_t *slot_pos,
                               int32_t *recv_src, void *recv,
                               float *recv_scale, void *ws, size_t ws_bytes,
                               int num_sms, int32_t *d_err, void *stream);

/*
 * ep_combine -- bring the expert outputs back to their tokens.
 *
 * DeepEP's combine (chinainews.com item, feature list; dataforcee.us
 * rewrite, "Technological Views and Benefits").  Reading: a gate-weighted
 * sum accumulated in fp32 in slot order:
 *   acc = 0.0f;  for j = 0..k-1 with slot_pos[t,j] = p >= 0:
 *       acc = fma(w[t,j], float(y[p, :]), acc)
 *   out[t, :] = bf16 round-to-nearest-even(acc)
 * y          [y_rows, H] bf16 expert outputs in receive-row order.
 * y_rows     rows of y (0 means T*k); slot rows outside [0, y_rows) are
 *            skipped.
 * slot_pos   [T,k] int32 (packed or aligned layout).
 * w          [T,k] fp32 gate weights (4-byte aligned), or NULL for unit
 *            weights: out[t] is then the plain fp32 sum of the kept slot
 *            rows (how per-rank partial outputs combine, see
 *            ep_get_rank_layout).
 * out        [T,H] bf16; a token with no kept slot gets +0.
 * Limits as ep_dispatch (H % 8 == 0).  num_sms and d_err as ep_dispatch.
 */
ep_status_t ep_combine(const void *y, int y_rows, int T, int H, int k,
                       const int32_t *slot_pos, const float *w, void *out,
                       int num_sms, int32_t *d_err, void *stream);

/*
 * ep_combine_fp8 -- ep_combine for expert outputs kept in the FP8 form of
 * the dispatch (e4m3 codes plus one fp32 scale per row and 128-channel
 * block).
 *
 * A combine variant beside DeepEP's FP8 dispatch (chinainews.com item,
 * feature list; Wallstreetcn review of the release): the pages give no
 * arithmetic for it.  Reading: each value is decoded exactly and scaled in
 * fp32, then enters the same chain as ep_combine:
 *   v = fp32_rn(e4m3(y_q[p, c]) * y_scale[p, c / 128])
 *   acc = fma(w[t,j], v, acc) in slot order from 0.0f; out = bf16_rne(acc)
 * y_q       [y_rows, H] e4m3 bytes (16-byte aligned).
 * y_scale   [y_rows, H/128] fp32 (4-byte aligned; under an SM budget,
 *           16-byte aligned rows and H % 512 == 0 take the bulk-copy
 *           kernel).
 * y_rows, slot_pos, w, out, num_sms, d_err: as ep_combine.  H % 128 == 0.
 */
ep_status_t ep_combine_fp8(const void *y_q, const float *y_scale, int y_rows,
                           int T, int H, int k, const int32_t *slot_pos,
                           const float *w, void *out, int num_sms,
                           int32_t *d_err, void *stream);

/*
 * ep_pad_layout -- receive segments aligned for a grouped GEMM.
 *
 * The dispatch layout packs the experts' rows back to back; a grouped GEMM
 * over the receive buffer in tiles of `align` rows wants each expert's
 * segment to start on a tile boundary.  The pages describe the layout only
 * as DeepEP's dispatch target (chinainews.com item, feature list); the
 * padded form is this library's.  From a layout of ep_get_layout:
 *   off_pad[e]        = sum_{e' < e} ceil(cnt_e[e'] / align) * align,
 *                       off_pad[E] = rows in use with padding
 *   slot_pos_pad[t,j] = off_pad[e] + (slot_pos[t,j] - off_e[e]), or -1
 *   recv_src_pad[r]   = token of row r; -1 for padding rows and past
 *                       off_pad[E]
 * cnt_e        [E] int32 and slot_pos [T,k] int32 from one ep_get_layout.
 * off_pad      [E+1] int32.  slot_pos_pad [T,k] int32 (may be slot_pos).
 * recv_src_pad [ep_aligned_rows(T, k, E, align)] int32.
 * Dispatch and combine then take slot_pos_pad with recv_rows = y_rows =
 * ep_aligned_rows(T, k, E, align).  T >= 0, k >= 1, 1 <= E <= EP_MAX_E,
 * align >= 1, T*k + E*(align-1) < 2^31.
 */
size_t ep_aligned_rows(int T, int k, int E, int align);
ep_status_t ep_pad_layout(const int32_t *cnt_e, const int32_t *slot_pos,
                          int T, int k, int E, int align, int32_t *off_pad,
                          int32_t *slot_pos_pad, int32_t *recv_src_pad,
                          void *stream);

/*
 * ep_get_rank_layout -- rows of the rank-deduplicated dispatch: one receive
 * row per (token, rank) pair instead of one per (token, expert).
 *
 * DeepEP's high-throughput ("normal") kernels send a token once to each
 * peer rank that hosts any of its experts (frogred8 blog, "Implementation
 * of SMs dedicated to network communication": one sender per NVLink peer;
 * chinainews.com item, "Technical Details": normal kernels for training
 * and prefill over NVLink and RDMA); the receiving rank then spreads it
 * over its local experts.  Here, from the token-in-rank mask of
 * ep_get_layout:
 *   rank_row[t,r] = off_r[r] + #{t' < t : in_rank[t',r]}  if in_rank[t,r],
 *                   else -1 (rows of one rank in ascending token order)
 *   rank_src[q]   = token of rank row q; -1 past off_r[R]
 *   cnt_r, off_r  = tokens per rank and their exclusive scan (the same
 *                   values ep_get_layout writes)
 * Rows per token drop from k to the number of distinct ranks among its
 * experts (at most min(k, R)).  The dispatch itself is ep_dispatch with
 * slot_pos = rank_row and k = R (R <= EP_MAX_K there); the matching combine
 * is ep_combine with slot_pos = rank_row, k = R and w = NULL, summing the
 * per-rank partial outputs (each already gate-weighted on its rank).
 *
 * in_rank   [T,R] uint8 (0 / nonzero), rank_row [T,R] int32,
 * rank_src  [T*R] int32, cnt_r [R], off_r [R+1] int32.
 * T >= 0, 1 <= R <= EP_MAX_R, T*R < 2^31.  ws / ws_bytes as ep_get_layout,
 * sized by ep_rank_layout_workspace_bytes (0 for T*R < 65536).
 */
size_t ep_rank_layout_workspace_bytes(int T, int R);
ep_status_t ep_get_rank_layout(const uint8_t *in_rank, int T, int R,
                               int32_t *cnt_r, int32_t *off_r,
                               int32_t *rank_row, int32_t *rank_src, void *ws,
                               size_t ws_bytes, void *stream);

/*
 * ep_map_replicas -- route the slots of busy experts to redundant copies.
 *
 * DeepSeek's expert load balancer places extra copies of the experts in
 * high demand (deepseekaiinsights, Open Source Week overview, "EPLB and
 * DualPipe"); the page names no rule for which copy serves a token.
 * Reading: the i-th slot of logical expert e in the dispatch layout's
 * stable token-major order (i = slot_pos[t,j] - off_e[e]) goes to copy
 * i mod n_e, so one expert's copies get equal shares to within one slot:
 *   phys_idx[t,j] = rep_ids[rep_off[e] + i mod (rep_off[e+1] - rep_off[e])]
 * A dropped slot stays -1; a bad id or an expert without copies is
 * recorded in d_err (EP_ERR_INDEX) and its slot dropped.  Lay out and
 * dispatch the physical ids with ep_get_layout(phys_idx, 0, T, k, E_phys,
 * R_phys, ...) and the rest of the path as usual.
 *
 * idx        [T,k] logical ids (int64 or int32, as ep_get_layout).
 * slot_pos   [T,k] and off_e [E+1] int32 from ep_get_layout of idx.
 * rep_off    [E+1] int32, nondecreasing; rep_ids [rep_off[E]] int32.
 * phys_idx   [T,k] int32 physical ids.
 * T >= 0, k >= 1, E >= 1, T*k < 2^31.
 */
ep_status_t ep_map_replicas(const void *idx, int idx_is_int64, int T, int k,
                            int E, const int32_t *slot_pos,
                            const int32_t *off_e, const int32_t *rep_off,
                            const int32_t *rep_ids, int32_t *phys_idx,
                            int32_t *d_err, void *stream);

/* Size of the scratch array behind ep_get_layout_noalloc (256 KiB). */
#define EP_NOALLOC_SCRATCH_BYTES (256u * 1024u)

/*
 * ep_get_layout_noalloc -- ep_get_layout for callers that cannot allocate
 * device memory.
 *
 * The DeepEP pages have no counterpart to this entry point; it exists for
 * deployments, not for the method.  Some callers cannot call cudaMalloc
 * or keep a workspace of their own: a runtime whose device memory is all
 * handed out up front by its own pool (an extra allocation would fail or
 * break its accounting), or a latency-critical loop that must not pay the
 * implicit device-wide synchronisation of cudaMalloc / cudaFree.  This
 * variant takes the same arguments as ep_get_layout minus ws / ws_bytes
 * and computes the same outputs.  Its scratch is a fixed array of
 * EP_NOALLOC_SCRATCH_BYTES bytes inside the library: every GPU that loads
 * the library holds one copy of it until the process exits, and the call
 * itself allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library routine).
 *
 * Limits: batches of up to 2^19 slots (T*k) use no scratch at all; a
 * larger batch whose tiled layout needs more scratch than the array
 * (ep_layout_workspace_bytes(T, k, E, R) > EP_NOALLOC_SCRATCH_BYTES, e.g.
 * 100000 tokens, top-8 over 1024 experts) is rejected with
 * EP_ERR_UNSUPPORTED and a message, before anything is enqueued.  For
 * example 70000 tokens, top-8 over 128 experts in 16 ranks needs 170 KB
 * and fits.
 *
 * Device: the array used is the current device's.  A call that uses it
 * (the tiled sizes) checks that `stream` belongs to the current device
 * and that idx is memory the current device can read, and returns
 * EP_ERR_INVALID_ARG otherwise, before anything is enqueued.
 *
 * Set-up: each call that uses the array looks up its device address
 * (cudaGetSymbolAddress) in the current context -- never a stale one,
 * whichever context is current.  The first lookup on a device loads the
 * library's module there; make that first call before any stream capture
 * begins.
 *
 * Sharing: every call on a device uses the same array, which keeps the
 * last call's contents (it is zero-filled when the module loads).  The
 * only part that must start at zero, the 16-byte ticket, is left at zero
 * by every call's own kernels, even after calls that overlapped; nothing
 * else is enqueued.  Calls whose work overlaps on the GPU (different
 * streams, no ordering between them) race on the array and give wrong
 * layouts: order them on one stream, or use ep_get_layout with one
 * workspace per stream.
 */
ep_status_t ep_get_layout_noalloc(const void *idx, int idx_is_int64, int T,
                                  int k, int E, int R, int32_t *cnt_e,
                                  int32_t *cnt_r, uint8_t *in_rank,
                                  int32_t *off_e, int32_t *off_r,
                                  int32_t *slot_pos, int32_t *recv_src,
                                  int32_t *d_err, void *stream);

/*
 * ep_debug_expire_first_wait -- testing switch for the bounded waits.
 *
 * The bulk-copy kernels (ep_combine with k <= 8 under an SM budget,
 * num_sms > 0, once its (token, 1 KB) items no longer fit 13 CTAs per
 * budgeted SM; ep_combine_fp8 with k <= 8; the FP8 ep_dispatch for
 * H % 512 == 0; both kernels of ep_layout_dispatch) wait for their own
 * asynchronous copies on shared-memory barriers, each wait bounded by an
 * iteration limit; when a limit
 * runs out the kernel records EP_ERR_TIMEOUT in d_err, waits (bounded) for
 * the copies it still has in flight and returns, leaving its output
 * incomplete.  With on != 0, the first such wait of every CTA of kernels
 * launched afterwards gives up at once, without polling, while its copy
 * still lands normally -- so that path can be run and checked without
 * making any copy fail.  The grid layout kernel (ep_get_layout for
 * 65536 <= T*k <= 2^19) waits the same way, bounded, at two barriers
 * between its CTAs; the switch makes the first of them give up at once in
 * every CTA that has not seen all CTAs arrive: such a CTA records
 * EP_ERR_TIMEOUT and places none of its slots, and the workspace's
 * counters are still left at zero.  on == 0 (the default) restores the
 * normal limits.  Process-wide; for tests only (the pages have no
 * counterpart).
 */
void ep_debug_expire_first_wait(int on);

/*
 * Waits for `stream` and returns the device error word *d_err (EP_OK when
 * no bad id was met), or EP_ERR_CUDA if the copy failed.
 */
ep_status_t ep_read_error(const int32_t *d_err, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_H_ */
