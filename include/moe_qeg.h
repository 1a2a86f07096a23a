/*
 * moe_qeg.h - union-of-experts 4-bit quantized MoE SwitchGLU layer for NVIDIA
 * B200 (sm_100a).  C ABI; plain pointers and sizes only.
 *
 * What the layer computes (per window of T tokens routed top-k over E experts):
 *   for every (token t, slot j) pair p = t*k + j with expert e = topk_idx[p]:
 *     g = bf16(Wg[e] x_t), v = bf16(Wu[e] x_t)   (fp32 accumulation)
 *     h = bf16(silu(g) * v)
 *     y = Wd[e] h                               (fp32)
 *   out[t] = bf16( sum_j topk_w[t, j] * y_(t, j) )
 * where each weight matrix is 4-bit affine quantized with groups of 64 input
 * columns: w = scale * q + bias, q in 0..15, scale and bias bf16.  This is the
 * SwitchGLU of the moe_bench.py script in "gather_qmm at M=1 streams 4-bit
 * expert weights at ~half the bandwidth of M=4" (mlx issue 4509, "Script":
 * up, gate, silu(gate)*up, down, mx.quantize group 64, bits 4, affine), with
 * the one-pass bf16(up)*silu(gate) epilogue of "Apple7/8 MoE gate and up in
 * one decode pass" (splash PR 45, "What changed").
 *
 * How: instead of streaming one expert block per (token, expert) pair, the
 * union of the routed experts is formed once and each distinct expert's
 * gate/up/down block is read from HBM once and applied to every pair routed to
 * it ("Small-L fused expert gather for fine-grained MoE decode", mlx discussion
 * 3801, first post "Two implications" item 1, and the sort-by-expert /
 * ragged-matmul framing of the second post).
 *
 * Layouts (row-major, all device memory, caller-owned):
 *   x          bf16 [T, hidden]
 *   topk_idx   int32 [T, k]       expert ids; ids outside [0, E) are skipped
 *                                 and flagged (see moe_read_device_status)
 *   topk_w     fp32 [T, k]        router weights, used as given
 *   wg_q, wu_q uint32 [E, inter, hidden/8]  (gate, up: rows = output features)
 *   wg_s/wg_b, wu_s/wu_b  bf16 [E, inter, hidden/64]
 *   wd_q       uint32 [E, hidden, inter/8]
 *   wd_s/wd_b  bf16 [E, hidden, inter/64]
 *   out        bf16 [T, hidden]
 * Element c of a weight row is nibble c % 8 (bits 4*(c%8) .. 4*(c%8)+3, least
 * significant first) of 32-bit word c / 8.  bf16 values are passed as their
 * raw 16-bit patterns (uint16_t).
 *
 * Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 * the legacy default stream).  They perform no host synchronisation, no
 * device allocation (except where stated) and no host-device copies.
 * Results are deterministic: the same inputs give the same bits on every run.
 */
#ifndef MOE_QEG_H
#define MOE_QEG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad multiple */
  MOE_ERR_UNSUPPORTED = 2,  /* shape outside the supported range, misaligned pointer */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_INDEX = 4, /* a kernel met an expert id outside [0, E) */
  MOE_ERR_TIMEOUT = 5,      /* a kernel's bounded wait ran out (internal error) */
  MOE_ERR_WORKSPACE = 6     /* workspace too small, or growth needed during capture */
} moe_status;

/* Supported range (checked on the host; violations return MOE_ERR_UNSUPPORTED):
 * hidden and inter multiples of 64, hidden <= 8192, inter <= 8192; E <= 1024;
 * T*k <= 65536.  Windows of more than 1024 pairs (or whose persistent-kernel
 * plan does not fit) take the grouped tensor-core path, which further needs
 * hidden a multiple of 256, inter a multiple of 128 and T*k <= 57856 (its
 * combine keeps a pair index per pair in shared memory); moe_select_path tells
 * which path a shape takes (0: the call returns MOE_ERR_UNSUPPORTED). */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_DIM 8192
#define MOE_MAX_PAIRS 65536

/* Human-readable name of a status code (static string). */
const char* moe_status_str(int status);

/* The CUDA runtime's message for the most recent MOE_ERR_CUDA returned on the
 * calling thread ("no error" if none); a static string. */
const char* moe_last_error(void);

/* Bytes of workspace that moe_switchglu_forward_ws needs for this shape
 * (0 on invalid arguments).  The workspace holds the kernel's progress
 * counters, the route-union arrays, h = bf16 [T*k, inter] and y = fp32
 * [T*k, hidden].  The counter region (the first moe_workspace_layout()[1]
 * bytes) must be zero before the first call on a buffer; every call leaves it
 * zero again (after a call that ends in MOE_ERR_TIMEOUT it must be zeroed
 * again).  Zeroing the whole buffer once is enough.  The rest is scratch. */
size_t moe_workspace_size(int T, int k, int E, int hidden, int inter);

/*
 * Route-union ("Small-L fused expert gather", mlx discussion 3801, second
 * post: sort the (position, expert) pairs by expert and stream each unique
 * expert once).  From topk_idx [T, k] (device) it writes (device):
 *   unique[min(E, T*k)]     distinct expert ids, ascending
 *   offsets[min(E, T*k)+1]  offsets[i] = number of pairs of unique[0..i);
 *                           offsets[u] = number of valid pairs
 *   pair_list[T*k]          pair ids p = t*k + j grouped by expert in the
 *                           order of `unique`, ascending p within an expert;
 *                           entries past offsets[u] are -1
 *   num_unique[1]           u
 * Entries of unique/offsets past u (resp. u+1) are left unchanged.  Pairs
 * with an id outside [0, E) are left out and flag MOE_ERR_DEVICE_INDEX.
 * All arrays must be 4-byte aligned.  Integer output, bit-exact.
 */
moe_status moe_route_union(const int32_t* topk_idx, int T, int k, int E, int32_t* unique,
                           int32_t* offsets, int32_t* pair_list, int32_t* num_unique,
                           void* stream);

/*
 * The fused union-of-experts SwitchGLU forward described at the top of this
 * file, using caller-provided device workspace of at least
 * moe_workspace_size(T, k, E, hidden, inter) bytes (16-byte aligned, counter
 * region zero as described there).  x, the weight arrays, out and workspace
 * must be 16-byte aligned; topk_idx and topk_w 4-byte aligned.  Tokens whose
 * pairs are all invalid get a zero output row.  The forward is one kernel of
 * one CTA per SM whose CTAs wait on one another's progress through counters
 * in the workspace (it is launched cooperatively, so all CTAs are resident);
 * two calls that share a workspace must not run concurrently.  Capturable in a
 * CUDA graph.
 */
moe_status moe_switchglu_forward_ws(const uint16_t* x, const int32_t* topk_idx,
                                    const float* topk_w, const uint32_t* wg_q,
                                    const uint16_t* wg_s, const uint16_t* wg_b,
                                    const uint32_t* wu_q, const uint16_t* wu_s,
                                    const uint16_t* wu_b, const uint32_t* wd_q,
                                    const uint16_t* wd_s, const uint16_t* wd_b, int T, int k,
                                    int E, int hidden, int inter, uint16_t* out, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * Same as moe_switchglu_forward_ws with a library-owned workspace per device.
 * The workspace is allocated (cudaMalloc) on the first call that needs more
 * than the current one; such a call must not be made during stream capture
 * (it returns MOE_ERR_WORKSPACE then).  The buffer lives until process exit.
 * Calls on different streams of one device share it and must not overlap.
 */
moe_status moe_switchglu_forward(const uint16_t* x, const int32_t* topk_idx, const float* topk_w,
                                 const uint32_t* wg_q, const uint16_t* wg_s,
                                 const uint16_t* wg_b, const uint32_t* wu_q,
                                 const uint16_t* wu_s, const uint16_t* wu_b,
                                 const uint32_t* wd_q, const uint16_t* wd_s,
                                 const uint16_t* wd_b, int T, int k, int E, int hidden,
                                 int inter, uint16_t* out, void* stream);

/*
 * Same layer as moe_switchglu_forward, with no allocation of any kind: the
 * scratch (progress counters, union arrays, h and y) is one fixed array of
 * MOE_STATIC_SCRATCH_BYTES (4 MiB) per device, a `__device__` global of the
 * library.  The pages describe no such entry point; it exists for callers that
 * may not allocate (allocator-free or pre-planned memory).
 *   - Limit: shapes whose moe_workspace_size exceeds MOE_STATIC_SCRATCH_BYTES
 *     return MOE_ERR_WORKSPACE and moe_last_error() says so.  4 MiB holds
 *     T*k <= 128 at hidden 4096 / inter 2048 (e.g. T <= 16 at top-8).
 *   - Set-up: the first call on each device looks up the array's address
 *     (cudaGetSymbolAddress, that device current) and caches it; make that
 *     first call before any stream capture.
 *   - Zeroing: each call clears the counter region (its first 4*1539 bytes)
 *     with cudaMemsetAsync on `stream` before the kernel; nothing else needs
 *     to start at zero.
 *   - Races: all calls on one device share the one array.  Calls that overlap
 *     (different streams, or host threads, without ordering between them)
 *     corrupt each other's results; order them on one stream or with events.
 * Arguments, alignment rules and results are those of moe_switchglu_forward_ws.
 */
#define MOE_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
moe_status moe_switchglu_forward_static(const uint16_t* x, const int32_t* topk_idx,
                                        const float* topk_w, const uint32_t* wg_q,
                                        const uint16_t* wg_s, const uint16_t* wg_b,
                                        const uint32_t* wu_q, const uint16_t* wu_s,
                                        const uint16_t* wu_b, const uint32_t* wd_q,
                                        const uint16_t* wd_s, const uint16_t* wd_b, int T, int k,
                                        int E, int hidden, int inter, uint16_t* out,
                                        void* stream);

/*
 * mxfp4 banks ("Small-L fused expert gather for fine-grained MoE decode", mlx
 * discussion 3801: GLM-5.2's routed banks are "mxfp4 gs32"; the pages define the
 * format no further, so the OCP microscaling reading is taken).  Per matrix:
 *   q  uint32 [E, rows, cols/8]   e2m1 codes, packed like the affine codes
 *                                 (element c = nibble c%8 of word c/8, LSB
 *                                 first); code bit 3 = sign, bits 2..0 index
 *                                 0, 0.5, 1, 1.5, 2, 3, 4, 6
 *   e  uint8  [E, rows, cols/32]  e8m0 scale bytes, 2^(e - 127) (255 = NaN)
 *   w  = e2m1(q) * 2^(e - 127), one scale per 32 consecutive columns.
 * Gate and up: rows = inter, cols = hidden; down: rows = hidden, cols = inter.
 * Everything else (x, topk_idx, topk_w, out, workspace rules, errors, capture)
 * is as for moe_switchglu_forward_ws / moe_switchglu_forward, with the workspace
 * sized by moe_workspace_size_mxfp4.  Small windows take the persistent kernel,
 * larger ones the grouped tensor-core path (moe_select_path_mxfp4 returns 1 or 2,
 * under the same shape rules as the affine format); a shape neither takes
 * (moe_select_path_mxfp4 returns 0) gives MOE_ERR_UNSUPPORTED.  On the grouped
 * path each weight e2m1(q) 2^(e - 127) is exact in bf16 and is the MMA's operand.
 */
size_t moe_workspace_size_mxfp4(int T, int k, int E, int hidden, int inter);
int moe_select_path_mxfp4(int T, int k, int E, int hidden, int inter);
moe_status moe_switchglu_forward_mxfp4_ws(const uint16_t* x, const int32_t* topk_idx,
                                          const float* topk_w, const uint32_t* wg_q,
                                          const uint8_t* wg_e, const uint32_t* wu_q,
                                          const uint8_t* wu_e, const uint32_t* wd_q,
                                          const uint8_t* wd_e, int T, int k, int E, int hidden,
                                          int inter, uint16_t* out, void* workspace,
                                          size_t workspace_bytes, void* stream);
moe_status moe_switchglu_forward_mxfp4(const uint16_t* x, const int32_t* topk_idx,
                                       const float* topk_w, const uint32_t* wg_q,
                                       const uint8_t* wg_e, const uint32_t* wu_q,
                                       const uint8_t* wu_e, const uint32_t* wd_q,
                                       const uint8_t* wd_e, int T, int k, int E, int hidden,
                                       int inter, uint16_t* out, void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word that the
 * kernels set instead of trapping: MOE_ERR_DEVICE_INDEX if an expert id was
 * out of range, MOE_ERR_TIMEOUT if a bounded wait ran out, else MOE_OK (or
 * MOE_ERR_CUDA if the synchronisation itself failed).  On MOE_ERR_TIMEOUT it
 * also zeroes the counter region of the workspace the library owns on the
 * current device (the one moe_switchglu_forward uses), so that later calls
 * start clean; work queued on other streams that uses that workspace must be
 * complete first.  A caller-owned workspace (moe_switchglu_forward_ws) is the
 * caller's to clear after a timeout.
 */
moe_status moe_read_device_status(void* stream);

/*
 * The limit of every bounded wait in the kernels (a spin on an mbarrier or on a
 * progress counter) on the current device, in nanoseconds: 0 restores the default of
 * 2 s; values below 1000 are raised to 1000; above 2 s is MOE_ERR_INVALID_ARG.  A
 * wait that runs out sets MOE_ERR_TIMEOUT in the error word and the kernel returns
 * (a shorter limit lets a watchdog, or a test, see a stalled call sooner).  The waits
 * that let copies and MMAs already in flight land before a CTA exits keep 2 s.  Takes
 * effect for kernels launched after it; synchronous with respect to the device.
 */
moe_status moe_set_wait_limit_ns(unsigned long long ns);

/*
 * Router step ahead of the layer (the routing of the tiny parity configuration:
 * top-k of softmax over the experts, renormalised over the k).  For each token t
 * of logits [T, E] (fp32, row-major, finite values): topk_idx[t, 0..k) = the k
 * experts with the largest logits, in descending logit order, the lower expert
 * id first among equal logits; topk_w[t, j] = exp(l_j - m) / D, m = the row's
 * largest logit, D = the sum of exp(l - m) over the k picks (renormalize != 0)
 * or over all E (renormalize == 0).  The outputs are the topk_idx / topk_w
 * arguments of moe_switchglu_forward.
 *   logits [T*E] fp32, topk_idx [T*k] int32, topk_w [T*k] fp32: device memory
 *   owned by the caller, 4-byte aligned.  One launch on `stream`, no host sync,
 *   capturable.
 * Errors: MOE_ERR_INVALID_ARG for null pointers, T, E or k <= 0, or k > E;
 * MOE_ERR_UNSUPPORTED for E > 1024, k > 32, T*k > MOE_MAX_PAIRS or a misaligned
 * pointer (nothing is launched); MOE_ERR_CUDA if the launch fails.
 */
moe_status moe_router_topk(const float* logits, int T, int E, int k, int renormalize,
                           int32_t* topk_idx, float* topk_w, void* stream);

/*
 * The router step and the layer in one call: the experts of each token are picked
 * from router logits exactly as moe_router_topk does (top-k of softmax, descending,
 * lower id first among equal logits, weights renormalised over the k when
 * renormalize != 0), then the layer of moe_switchglu_forward_ws runs on those picks.
 * On the persistent path (moe_select_path == 1 with the picks' shared-memory room)
 * every CTA makes the picks in its own prologue, so there is one launch for the
 * router and the layer; on the grouped path the router kernel runs first (two
 * launches more than the layer's own).  Both write the picks and weights to
 * topk_idx / topk_w ([T*k] int32 / fp32, device, 4-byte aligned, caller-owned),
 * which equal moe_router_topk's on the same logits bit for bit.
 *   logits [T*E] fp32 (finite), x, bank and out as for moe_switchglu_forward_ws;
 *   workspace of moe_workspace_size(T, k, E, hidden, inter) bytes.
 * "Small-L fused expert gather for fine-grained MoE decode" (mlx discussion 3801):
 * the picks feed the union of the window directly.
 * Errors: those of moe_switchglu_forward_ws and moe_router_topk (E > 1024 or k > 32
 * is MOE_ERR_UNSUPPORTED, k > E is MOE_ERR_INVALID_ARG).
 */
moe_status moe_switchglu_forward_routed_ws(
    const uint16_t* x, const float* logits, int renormalize, const uint32_t* wg_q,
    const uint16_t* wg_s, const uint16_t* wg_b, const uint32_t* wu_q, const uint16_t* wu_s,
    const uint16_t* wu_b, const uint32_t* wd_q, const uint16_t* wd_s, const uint16_t* wd_b, int T,
    int k, int E, int hidden, int inter, uint16_t* out, int32_t* topk_idx, float* topk_w,
    void* workspace, size_t workspace_bytes, void* stream);

/* moe_switchglu_forward_routed_ws with a library-owned workspace per device (as for
 * moe_switchglu_forward). */
moe_status moe_switchglu_forward_routed(const uint16_t* x, const float* logits, int renormalize,
                                        const uint32_t* wg_q, const uint16_t* wg_s,
                                        const uint16_t* wg_b, const uint32_t* wu_q,
                                        const uint16_t* wu_s, const uint16_t* wu_b,
                                        const uint32_t* wd_q, const uint16_t* wd_s,
                                        const uint16_t* wd_b, int T, int k, int E, int hidden,
                                        int inter, uint16_t* out, int32_t* topk_idx,
                                        float* topk_w, void* stream);

/*
 * Which kernel path a call with this shape takes, without launching anything:
 * 1 = expert-major dequant-GEMV layer kernel (T*k <= 1024 and its shared-memory
 * plan fits), 2 = grouped tensor-core path (route-union, x packing, gate+up and
 * down GEMMs on tcgen05, combine: five launches; hidden % 256 == 0 and
 * inter % 128 == 0), 0 = invalid or unsupported shape.  The workspace size
 * (moe_workspace_size) follows the path: path 2 adds the packed activations,
 * about 2*(hidden+inter)*(T*k + 15*min(E, T*k)) bytes.
 */
int moe_select_path(int T, int k, int E, int hidden, int inter);

/*
 * Offsets (bytes) of the workspace regions for this shape, for inspection in
 * tests: out[0] = progress counters (zero between calls; they end where
 * out[1] starts), out[1] = num_unique (int32), out[2] =
 * unique, out[3] = offsets, out[4] = pair_list, out[5] = h (bf16 [T*k, inter]
 * in pair_list order), out[6] = y (fp32 [T*k, hidden] in pair_list order),
 * out[7] = total bytes.  Returns MOE_ERR_INVALID_ARG on bad shapes.
 */
moe_status moe_workspace_layout(int T, int k, int E, int hidden, int inter, size_t out[8]);

#ifdef __cplusplus
}
#endif

#endif /* MOE_QEG_H */
