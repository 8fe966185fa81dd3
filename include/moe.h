/*
 * moe.h - C ABI of libmoe.so: the Mixture-of-Experts layer forward on one B200 (sm_100a),
 *         "route + pack + compute + combine".
 *
 * The operation ("271,104 Routes: What I Missed About Mixture-of-Experts", sections 1-3;
 * "Mixture of Experts: Routing, Dispatch, and Load Balancing", sections 2-4):
 *   z      = x W_r^T + bias                          router logits        [T, E]
 *   ids, g = top-k of z, gate weights (3 modes)      routing              [T, k]
 *   pack   = rows of x duplicated per kept route and grouped by expert   [R, d]
 *   H      = SiLU(X_p Wg_e^T) * (X_p Wu_e^T)         per expert segment   [R, F]
 *   Y      = H Wd_e^T                                per expert segment   [R, d]
 *   y[t]   = sum_j g[t,j] Y[row(t,j)] (+ shared expert) (+ x[t])          [T, d]
 *
 * Conventions shared by every entry point
 *   Memory      Every pointer argument is a DEVICE pointer owned by the caller unless
 *               stated otherwise.  The library never allocates device memory.
 *   Layout      Row-major, densely packed.  Weights use nn.Linear storage [out, in]
 *               ("Mixture of Experts: Routing, Dispatch, and Load Balancing", section 1:
 *               the math form W_router [d, N] is stored as [N, d]); per-expert weights
 *               are stacked along a leading expert axis.
 *   Types       dtype MOE_BF16: x, weights, packed rows, H, Y and y are bf16 (fp32
 *               accumulation).  dtype MOE_F32: all of those are fp32.  Gates and the
 *               logit bias are always fp32; ids, rows and offsets are int32.
 *   Streams     Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *               default stream).  Host-side validation errors are returned at once and
 *               nothing is launched.  Errors found on the device (bad expert id, a
 *               bounded wait that ran out) are recorded in the status word at the start
 *               of the workspace; read it with moe_get_device_status.
 *   Workspace   `ws` is caller-owned device memory of at least moe_workspace_bytes(cfg)
 *               bytes, 256-byte aligned.  Its first 256 bytes must be zero before first
 *               use (moe_workspace_init does this).  Calls that share a workspace must be
 *               ordered on one stream.
 *   Determinism The same inputs give bit-identical outputs (no floating-point atomics;
 *               packed positions come from an ordered count, not from atomic arrival).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Compatible with cudaStream_t without including CUDA headers. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,        /* null pointer, non-positive size, k > E, bad enum       */
  MOE_ERR_UNSUPPORTED = 2,    /* valid but outside what the kernels handle (see below)   */
  MOE_ERR_WORKSPACE = 3,      /* workspace null or misaligned                             */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call or a launch failed            */
  MOE_ERR_BAD_EXPERT_ID = 5,  /* device: an id outside [0, E) or repeated within a token  */
  MOE_ERR_TIMEOUT = 6         /* device: a bounded wait ran out; the kernel returned early */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Where the softmax sits ("MoE Inference Visualized", The Router; "Mixture of Experts:
 * Routing, Dispatch, and Load Balancing", section 3; "Mixture-of-experts routing",
 * The gate).  Ranking is always on the logits, ties to the lower expert index.     */
typedef enum {
  MOE_GATE_SOFTMAX_TOPK = 0,        /* g = softmax over all E, taken at the top-k        */
  MOE_GATE_SOFTMAX_TOPK_RENORM = 1, /* ... divided by the sum over the top-k             */
  MOE_GATE_TOPK_SOFTMAX = 2         /* g = softmax over the k selected logits only       */
} moe_gate_mode;

/* Where kept routes' rows go ("Mixture-of-Experts: routing and capacity", Capacity and its
 * Visual support: the dispatch buffer [E, C, d]).                                      */
typedef enum {
  MOE_LAYOUT_RAGGED = 0, /* expert segments packed back to back: R rows in total          */
  MOE_LAYOUT_PADDED = 1  /* expert e owns rows e*C .. e*C + C - 1 (needs capacity >= 0)    */
} moe_layout;

/* What happens to a route that finds its expert full ("Mixture-of-Experts: routing and
 * capacity", Overflow policies).                                                       */
typedef enum {
  MOE_OVERFLOW_DROP = 0,    /* the route is lost; the token keeps its other gates as they are */
  MOE_OVERFLOW_REROUTE = 1  /* the route moves to the token's next-best expert with a free
                             * slot (MOE_LAYOUT_PADDED only; see moe_dispatch)              */
} moe_overflow;

/* Tile shape of the bf16 expert-FFN GEMMs (the fp32 configuration ignores it).  All give
 * the same products; they differ in how ragged expert segments are padded and in how many
 * operand bytes each SM stages per k-block.                                               */
typedef enum {
  MOE_TILES_AUTO = 0,    /* row tiles over SM pairs when the routed experts average at
                          * least 512 rows each (C rows with the padded layout, else
                          * min(C, T k / E)) and d % 256 == 0, d_ff % 128 == 0; else row
                          * tiles, with a shared expert of T >= 512 rows on row tiles over
                          * SM pairs in launches of its own (moe_ffn_launches); column
                          * tiles when a fused step is requested                           */
  MOE_TILES_ROWS = 1,    /* 128 tokens x 256 output columns per tile: tokens on the MMA's M
                          * side; a segment is padded to a multiple of 128 rows           */
  MOE_TILES_COLUMNS = 2, /* 128 weight rows x up to 128 tokens per tile: weights on M,
                          * tokens on N; a segment is padded to a multiple of 16 rows     */
  MOE_TILES_PAIRS = 3,   /* column tiles over a pair of SMs (one M = 256 MMA, each SM
                          * holding half of the token tile); a segment is padded to a
                          * multiple of 32 rows; needs d and d_ff multiples of 256, else
                          * row tiles run                                                  */
  MOE_TILES_ROW_PAIRS = 4 /* row tiles over a pair of SMs: 256 tokens x 256 output columns
                          * per pair tile (one M = 256 MMA; each SM holds 128 tokens and
                          * half of the weight rows); a segment is padded to a multiple of
                          * 256 rows; needs d % 256 == 0 and d_ff % 128 == 0, else row
                          * tiles run                                                      */
} moe_tiles;

/* Steps of moe_forward fused into the expert GEMMs (bit flags; bf16, column tiles, drop
 * overflow policy; the staged calls ignore them).  The results are bit-identical to the
 * unfused path.  Source: "271,104 Routes...", section 3 (duplicate the token rows, group
 * them by expert, run the experts, undo the grouping): the copies into and out of the
 * grouped order are what these flags remove.                                          */
typedef enum {
  MOE_FUSE_NONE = 0,
  MOE_FUSE_GATHER = 1,  /* the gate/up GEMM reads each expert's token rows straight from x
                         * (by row_token); the pack writes only the route table          */
  MOE_FUSE_COMBINE = 2  /* the down GEMM's epilogue finishes each output row (gate-weighted
                         * sum in slot order, shared expert, residual) as soon as its last
                         * contribution is written; there is no separate combine launch   */
} moe_fuse;

typedef struct {
  int32_t T;            /* tokens in this call (>= 1)                                   */
  int32_t d;            /* model width                                                   */
  int32_t E;            /* routed experts, 1..256                                        */
  int32_t k;            /* experts per token, 1..min(E, 32)                              */
  int32_t d_ff;         /* expert hidden width F                                         */
  int32_t dtype;        /* moe_dtype                                                     */
  int32_t gate_mode;    /* moe_gate_mode                                                 */
  int32_t capacity;     /* < 0: dropless; else C >= 0 rows per expert (see moe_capacity) */
  int32_t has_shared;   /* 1: one always-on shared expert, gate 1, never dropped          */
  int32_t add_residual; /* 1: y = x + MoE(x)                                              */
  int32_t stats;        /* 1: the router also sums each token's full softmax per token
                         *    tile into the workspace, for moe_routing_stats; 0: off     */
  int32_t layout;       /* moe_layout                                                    */
  int32_t overflow;     /* moe_overflow                                                  */
  int32_t tiles;        /* moe_tiles (0 = automatic)                                     */
  int32_t fuse;         /* moe_fuse flags (0 = none); any flag selects column tiles and
                         * needs MOE_BF16 and MOE_OVERFLOW_DROP (else MOE_ERR_UNSUPPORTED);
                         * MOE_TILES_ROWS or MOE_TILES_ROW_PAIRS with a flag is
                         * MOE_ERR_INVALID                                                */
} moe_config;
/* Supported shapes (else MOE_ERR_UNSUPPORTED): bf16 needs d % 128 == 0 and
 * d_ff % 128 == 0; fp32 needs d % 4 == 0 and d_ff % 4 == 0.                            */

/* Capacity C = ceil(phi * T * k / E), phi = phi_num / phi_den, in exact integer
 * arithmetic ("Mixture-of-experts routing", Capacity; "Mixture-of-Experts: routing and
 * capacity", Capacity: ceil(8*2/4 * 1.25) = 5).  Returns -1 on invalid arguments.      */
int32_t moe_capacity(int32_t T, int32_t k, int32_t E, int32_t phi_num, int32_t phi_den);

/* Rows of the packed buffer: T*k, or E*C when capacity >= 0 and that is smaller
 * (MOE_LAYOUT_RAGGED); E*C (MOE_LAYOUT_PADDED).  Buffers of packed rows (x_packed,
 * row_token) need this many rows; H and y_packed need moe_max_rows + T rows when
 * has_shared (the shared expert's rows follow the routed ones).                        */
int64_t moe_max_rows(const moe_config* cfg);

/* Bytes of workspace that moe_forward needs (it keeps every intermediate there); the
 * staged calls need only the leading scratch part, which this also covers.
 * Returns 0 for an invalid config.                                                      */
size_t moe_workspace_bytes(const moe_config* cfg);

/* The FFN tile shape a config runs with: one of MOE_TILES_ROWS .. MOE_TILES_ROW_PAIRS
 * (cfg->tiles when its shape requirements hold, else row tiles; the automatic choice when
 * it is MOE_TILES_AUTO); 0 for an invalid config.  Host-only.                            */
int32_t moe_ffn_tile_shape(const moe_config* cfg);

/* Kernel launches of the expert FFN (moe_expert_ffn, and that step of moe_forward) for the
 * config: 2 (gate/up with SwiGLU, then down), or 4 when the automatic choice runs a shared
 * expert of at least 512 rows (T >= 512) on row tiles over SM pairs, in launches of its own,
 * while the routed segments take row tiles; 0 for an invalid config.  Host-only.          */
int32_t moe_ffn_launches(const moe_config* cfg);

/* Zero the status word and scratch header of a workspace (async on `stream`).          */
moe_status moe_workspace_init(void* ws, moe_stream_t stream);

/* Route: z = x W_r^T + bias, top-k ids (descending logit, ties to the lower index) and
 * gates ("271,104 Routes...", section 2 The Router; "Mixture-of-Experts: routing and
 * capacity", Router / Top-k and mixture).
 *   x         [T, d]  dtype          w_router [E, d] dtype      logit_bias [E] fp32 or NULL
 *   ids       [T, k]  int32 (out)    gates    [T, k] fp32 (out), slot j = j-th largest   */
moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router,
                     const float* logit_bias, int32_t* ids, float* gates, void* ws,
                     moe_stream_t stream);

/* Pack: per-expert demand, arrival-order positions (token order), capacity mask and
 * the expert-major packed copy of x ("271,104 Routes...", section 3 Dispatch, and its
 * subsection on capacity; "Mixture-of-Experts: routing and capacity", Worked case).
 *   ids        [T, k] int32 (in; ids outside [0,E) or repeated in a token are dropped and
 *              flagged MOE_ERR_BAD_EXPERT_ID in the status word)
 *   gates      [T, k] fp32 (in/out) with MOE_OVERFLOW_REROUTE, else unused (may be NULL)
 *   x_packed   [moe_max_rows, d] dtype (out): the p-th kept route of expert e (tokens
 *              ascending) is row offsets[e] + p, holding x[t]
 *   row_token  [moe_max_rows] int32 (out): token of each packed row
 *   route_row  [T, k] int32 (out): packed row of route (t, j), -1 when dropped
 *   offsets    int32 (out), the segment table.  MOE_LAYOUT_RAGGED: [E + 2], segment starts;
 *              offsets[E] = R (kept routes); offsets[E+1] = R + T with a shared expert,
 *              else R.  MOE_LAYOUT_PADDED: [2E + 2]: offsets[e] = e*C (e <= E),
 *              offsets[E+1] = E*C (+ T with a shared expert), offsets[E+2+e] = filled
 *              slots of expert e.  Rows of x_packed past an expert's filled slots are
 *              not written.
 *   demand     [E] int32 (out): routes asking for each expert before capacity
 * MOE_OVERFLOW_REROUTE ("Overflow policies": the overflowing route is handled by the
 * next-best expert by score): after the arrival-order pass, the routes that overflowed
 * are taken in arrival order; each moves to the best-ranked expert (logit descending,
 * ties to the lower index) that its token does not already hold and that has a free
 * slot, taking the next free slot; with none it is dropped.  A token with a moved route
 * gets its gates re-evaluated by the gate mode over its final experts (written to
 * `gates`); other tokens' gates are untouched.  The ranking reads the logits that
 * moe_route (or moe_forward) left in `ws` for the same config, so `ids` must come from
 * that call.  The expert that handles route (t, j) is route_row[t, j] / C.             */
moe_status moe_dispatch(const moe_config* cfg, const void* x, const int32_t* ids,
                        float* gates, void* x_packed, int32_t* row_token, int32_t* route_row,
                        int32_t* offsets, int32_t* demand, void* ws, moe_stream_t stream);

/* Compute: the SwiGLU expert FFNs as grouped GEMMs over the expert segments
 * ("MoE Inference Visualized", Expert Execution: down(SiLU(gate(x)) * up(x));
 * "271,104 Routes...", section 3: one dense matmul per expert batch).
 *   x          [T, d] (A operand of the shared expert; may be NULL without one)
 *   x_packed   [moe_max_rows, d]       offsets: the segment table of moe_dispatch
 *              (device; with MOE_LAYOUT_PADDED only the filled slots are computed)
 *   w_gate, w_up [E, F, d]   w_down [E, d, F]
 *   shared_gate, shared_up [F, d], shared_down [d, F]: NULL unless has_shared
 *   h          [moe_max_rows (+T), F] dtype (out, intermediate SiLU(g)*u)
 *   y_packed   [moe_max_rows (+T), d] dtype (out); the shared expert's row for token t
 *              is offsets[E] + t.  Rows past offsets[E+1] are not written.              */
moe_status moe_expert_ffn(const moe_config* cfg, const void* x, const void* x_packed,
                          const int32_t* offsets, const void* w_gate, const void* w_up,
                          const void* w_down, const void* shared_gate, const void* shared_up,
                          const void* shared_down, void* h, void* y_packed, void* ws,
                          moe_stream_t stream);

/* Combine: y[t] = sum_{j kept} gates[t,j] * y_packed[route_row[t,j]], summed in slot order
 * in fp32, + y_packed[offsets[E] + t] with a shared expert, + x[t] with add_residual
 * ("271,104 Routes...", section 1: y = sum p_i E_i(x); section 3: apply the gate weights
 * and restore the original token order; "Mixture-of-Experts: routing and capacity",
 * Top-k and mixture: output = weighted sum + shared + residual).
 *   residual   [T, d] (x) or NULL unless add_residual     y [T, d] dtype (out)           */
moe_status moe_combine(const moe_config* cfg, const void* y_packed, const int32_t* route_row,
                       const float* gates, const int32_t* offsets, const void* residual,
                       void* y, moe_stream_t stream);

/* The whole layer in one call: route -> pack -> compute -> combine, all intermediates in
 * `ws`, no host synchronisation.  ids_out / gates_out / demand_out / offsets_out are
 * optional copies of the routing metadata ([T,k], [T,k], [E], [E+2]; NULL to skip).    */
moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* logit_bias, const void* w_gate, const void* w_up,
                       const void* w_down, const void* shared_gate, const void* shared_up,
                       const void* shared_down, void* y, int32_t* ids_out, float* gates_out,
                       int32_t* demand_out, int32_t* offsets_out, void* ws,
                       moe_stream_t stream);

/* moe_forward that also records caller-created CUDA events (cudaEvent_t handles, e.g.
 * created with timing enabled) on `stream` around its kernels, for live per-kernel timing:
 * events[0] before the first kernel, events[i] after step i, i = 1..5 in the order
 * route, pack (with the reroute policy's kernels), gate/up GEMM, down GEMM, combine, for
 * n_events = 6; with n_events = 7 the reroute gets its own step after the pack (route,
 * pack, reroute, gate/up, down, combine; an empty interval without the reroute policy).
 * Any other n_events, or a NULL handle, is MOE_ERR_INVALID.                             */
moe_status moe_forward_profiled(const moe_config* cfg, const void* x, const void* w_router,
                                const float* logit_bias, const void* w_gate, const void* w_up,
                                const void* w_down, const void* shared_gate,
                                const void* shared_up, const void* shared_down, void* y,
                                int32_t* ids_out, float* gates_out, int32_t* demand_out,
                                int32_t* offsets_out, void* const* events, int32_t n_events,
                                void* ws, moe_stream_t stream);

/* Synchronise `stream`, copy the device status word of `ws` to *status_out (a moe_status)
 * and, if clear != 0, reset it to MOE_OK.  Returns MOE_ERR_CUDA if the copy fails.      */
moe_status moe_get_device_status(void* ws, moe_stream_t stream, int32_t clear,
                                 int32_t* status_out);

/* Test hook for failure detection: launch one CTA that waits on an mbarrier nothing
 * arrives at, bounded by `limit_ns` nanoseconds (1e3..1e10).  The wait runs out, the
 * kernel records MOE_ERR_TIMEOUT in the status word of `ws` and returns normally, so
 * the context stays usable.  It exercises the same bounded-wait routine the GEMM uses. */
moe_status moe_debug_bounded_wait(void* ws, int64_t limit_ns, moe_stream_t stream);

/* moe_dispatch without a workspace, for callers that cannot allocate device memory:
 * plugins that receive only their input and output buffers from a framework that owns
 * all device memory, runtimes with a memory budget fixed before start-up, or hot paths
 * that must not call an allocator (allocation may synchronise or take a global lock).
 * The pages have no counterpart; it is the pack step of moe_dispatch with the same
 * arguments and outputs, minus `gates` and `ws`.
 *   Scratch: the per-token-tile expert histogram lives in a fixed 64 KiB array inside the
 *   library (16384 int32 entries, held by every device that loads the library until the
 *   process exits).  Configurations whose histogram, ceil(T / tile) * E entries with the
 *   token tile of moe_dispatch, exceeds 16384 entries are rejected with
 *   MOE_ERR_UNSUPPORTED; nothing is launched then.
 *   Set-up: every call looks up the array's device address in the current device's
 *   context (a host-side query that enqueues no work), so the address stays right after
 *   cudaDeviceReset or under another context on the same device.  The first call on a
 *   device may load the library's device code for that context: make that first call
 *   before any stream capture.
 *   Sharing: every call on a device uses the same array and it keeps the last call's
 *   contents; nothing in it needs to start at zero because each call rewrites the entries
 *   it reads.  Calls that overlap on the GPU (other streams, other host threads) race on
 *   the array: order them on one stream.
 *   status: device int32 or NULL.  If given, it must hold 0 before the call; a bad expert
 *   id is recorded there as MOE_ERR_BAD_EXPERT_ID (the route is dropped).
 * Calls no cudaMalloc, cudaFree or other allocating routine.                            */
moe_status moe_dispatch_noalloc(const moe_config* cfg, const void* x, const int32_t* ids,
                                void* x_packed, int32_t* row_token, int32_t* route_row,
                                int32_t* offsets, int32_t* demand, int32_t* status,
                                moe_stream_t stream);
/*   (MOE_OVERFLOW_REROUTE needs the router's logits in a workspace: it is rejected here
 *   with MOE_ERR_UNSUPPORTED; both layouts are supported with MOE_OVERFLOW_DROP.)      */

/* Routing statistics of one layer call, written by moe_routing_stats (device memory). */
typedef struct {
  float aux_loss;        /* alpha * E * sum_e f_e * P_e                                      */
  float imbalance;       /* max_e demand_e / mean_e demand_e; 0 when no route is valid       */
  float drop_rate;       /* (T*k - kept) / (T*k)                                             */
  float padding_rate;    /* (E*C - kept) / (E*C) with capacity C > 0; 0 when dropless, C = 0 */
  int32_t kept;          /* kept routes R: offsets[E] (ragged), sum of filled slots (padded) */
  int32_t dropped;       /* T*k - R                                                          */
  int32_t max_demand;    /* max_e demand_e                                                   */
  int32_t busiest_expert;/* lowest e with demand_e = max_demand                              */
} moe_routing_summary;

/* Routing statistics of the last routed call on `ws`: the load-balancing terms and the
 * capacity outcome ("Mixture of Experts: Routing, Dispatch, and Load Balancing", section 4:
 * loss_aux = alpha * N * sum_i f_i P_i with f_i the fraction of tokens dispatched to
 * expert i and P_i the mean router probability; "Mixture-of-experts routing", Load
 * imbalance: I = max_e D_e / mean_e D_e; "Mixture-of-Experts: routing and capacity",
 * Worked case: drops and empty slots of the E x C buffer).
 *   f_e = demand_e / (T k): routes asking for e before capacity (with top-k each route
 *         counts once, so sum_e f_e = 1 when every id is valid).
 *   P_e = (1/T) sum_t softmax(z_t)_e over all E experts, whatever the gate mode.
 * With MOE_LAYOUT_PADDED, kept routes are the filled slots (after a reroute, if any).
 * Requires cfg->stats = 1 for the moe_route or moe_forward call that routed on this
 * workspace (its per-tile probability sums are read from `ws`; MOE_ERR_INVALID if
 * cfg->stats is 0).  Sums run in a fixed order (fp32 within a 128-token tile, fp64 across
 * tiles), so repeated calls give identical bits.
 *   demand   [E] int32, offsets [E+2] int32: from moe_dispatch, or moe_forward's
 *            demand_out / offsets_out.  NULL: the copies moe_forward keeps in `ws` when its
 *            own *_out argument was NULL.
 *   alpha    weight of the auxiliary value (1e-2 in the Switch Transformer setup).
 *   f, P     [E] fp32 (out, device) or NULL.     summary: one moe_routing_summary (out,
 *            device), required.                                                        */
moe_status moe_routing_stats(const moe_config* cfg, const int32_t* demand,
                             const int32_t* offsets, float alpha, float* f, float* P,
                             moe_routing_summary* summary, void* ws, moe_stream_t stream);

/* Static string for a status code. */
const char* moe_status_string(moe_status s);

/* Library version, for the binding's load check. */
int32_t moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
