/*
 * moe_layer.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts layer
 * over 4-bit block-quantised experts.
 *
 * One layer forward:
 *   router GEMM (fp32 logits) -> softmax top-k with renormalised gates ->
 *   token-to-expert permutation -> SwiGLU expert FFN read straight from
 *   MXFP4 / NVFP4 bytes -> gate-weighted combine (+ optional bf16 shared expert).
 * Experts are addressed through a resident-slot table: a budget of experts
 * lives in HBM slots, every expert lives in a library-owned pinned host
 * store, and experts a forward needs that are not resident are copied from
 * the pinned store with cudaMemcpyAsync on a side stream.
 *
 * Where each operation is defined (pages of the Strata reference set):
 *  - expert formats: "ro99/strata", "MXFP4 is read as MXFP4" (two E2M1 codes
 *    per byte, one E8M0 exponent per group of 32) and its model table
 *    ("NVFP4 or MXFP4 experts");
 *  - scale admission: "ro99/strata", "Scales are admitted, not clamped"
 *    (E8M0 codes 0 and 255 fail admission at load);
 *  - routing semantics, expert count and top-k come from the checkpoint and
 *    never change silently; exact mode completes or fails ("ro99/strata",
 *    list of rules under the introduction);
 *  - the paging hierarchy (every expert pinned in host RAM, a budget of hot
 *    experts on the GPU, shared experts always resident): "Strata, Explained",
 *    section 2, and strata.amperor.ai ("budget ... resident experts/layer");
 *  - paged output bit-identical to the resident model: strata.amperor.ai,
 *    legend of the memory-fit list.
 * The pages print no layer formula; the forms used (softmax routing,
 * h = silu(gate) * up, low nibble = even element, groups along the input
 * dimension) are the plainest readings and are listed in the design notes.
 *
 * Conventions for every call:
 *  - Nothing throws across this ABI.  Every call returns a moe_status_t; on
 *    failure moe_last_error() returns a thread-local description.
 *  - "stream" is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  All device work of a call is ordered on that stream: work the
 *    layer runs on a stream of its own (staging copies, the shared expert of
 *    a decode-sized forward) starts after the work queued on `stream` before
 *    the call and is joined back into `stream` before the call returns, so
 *    work queued on `stream` after the call follows all of it.
 *  - Device pointers are CUDA device memory of the layer's device; host
 *    pointers are ordinary (pageable or pinned) host memory.
 */
#ifndef MOE_LAYER_H
#define MOE_LAYER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_layer *moe_layer_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad pointer, size, shape or enum value            */
  MOE_ERR_ADMISSION = 2,   /* a block-scale code the format cannot represent   */
  MOE_ERR_SLOT_TABLE = 3,  /* slot out of range, duplicate slot, over budget    */
  MOE_ERR_OOM = 4,         /* device or pinned host allocation failed           */
  MOE_ERR_CUDA = 5,        /* a CUDA runtime call failed (detail in last_error) */
  MOE_ERR_UNSUPPORTED = 6  /* valid request this build does not implement       */
} moe_status_t;

/* Expert weight formats ("ro99/strata", model table: "NVFP4 or MXFP4
 * experts", "INT4 group-128, W4A16", "FP8 E4M3 block-128 with F32 inverse
 * scales"; never below four bits):
 *   MXFP4     E2M1 codes, two per byte, one E8M0 exponent per 32 along K;
 *   NVFP4     E2M1 codes, one E4M3 scale per 16 along K, one fp32 scale per
 *             matrix;
 *   INT4G128  signed 4-bit integers (two's complement, -8..7), two per byte,
 *             one bf16 scale per 128 along K; w = q * s;
 *   FP8B128   one E4M3 byte per weight, one fp32 inverse scale per block of
 *             128 rows x 128 columns; w = q * s.
 * In every format the even input index is the low nibble / first byte. */
typedef enum { MOE_FMT_MXFP4 = 0, MOE_FMT_NVFP4 = 1, MOE_FMT_INT4G128 = 2, MOE_FMT_FP8B128 = 3 } moe_fmt_t;

/* EXACT (default): activations stay 16-bit, FP4 weights decode exactly, fp32
 * accumulation.  A4 (opt-in): activations are quantised to the experts' own
 * 4-bit format before each expert GEMM so the tcgen05 block-scaled FP4 MMA can
 * run; never chosen silently. */
typedef enum { MOE_NUMERICS_EXACT = 0, MOE_NUMERICS_A4 = 1 } moe_numerics_t;

/* Router scoring: softmax over every routing target, or an independent
 * logistic per target (ids are the k largest logits either way). */
typedef enum { MOE_SCORING_SOFTMAX = 0, MOE_SCORING_SIGMOID = 1 } moe_scoring_t;

typedef enum { MOE_OUT_F32 = 0, MOE_OUT_BF16 = 1 } moe_out_dtype_t;

/* The routing semantics are what the checkpoint declares ("ro99/strata",
 * rules list: precision, routing, expert count and top-k come from the
 * checkpoint and never change silently): scoring, renormalisation, sink
 * targets (its model table has "256 experts + 2 sinks") and a sigmoid gate on
 * the shared expert are configuration, never chosen by the library.
 * Routing targets are the E experts followed by n_sinks sinks; a sink is
 * scored and chosen like an expert but has no FFN: choosing it adds nothing to
 * y (its gate share is not given to the other experts unless renormalisation
 * already did). */
typedef struct {
  int32_t hidden;       /* H; multiple of 256                                   */
  int32_t inter;        /* I (routed expert intermediate); multiple of 128       */
  int32_t n_experts;    /* E routed experts, 1..1024                            */
  int32_t top_k;        /* k, 1..min(E + n_sinks, 32)                           */
  int32_t shared_inter; /* I_s of the always-on bf16 shared expert, 0 = none;   */
                        /* multiple of 128                                      */
  int32_t fmt;          /* moe_fmt_t                                            */
  int32_t renormalize;  /* 1: the k chosen scores are divided by their sum;     */
                        /* 0: they are used as they are                         */
  int32_t numerics;     /* moe_numerics_t                                       */
  int32_t n_slots;      /* S resident HBM slots, 0..E                           */
  int32_t max_tokens;   /* largest T accepted by moe_forward, >= 1              */
  int32_t n_staging;    /* staging buffers for non-resident experts; >= 2 when  */
                        /* S < E (0 = library default)                          */
  int32_t device;       /* CUDA device ordinal                                   */
  int32_t scoring;      /* moe_scoring_t                                        */
  int32_t n_sinks;      /* sink targets after the experts, >= 0;                */
                        /* E + n_sinks + shared_gate <= 1024                    */
  int32_t shared_gate;  /* 1: the shared expert is scaled by                    */
                        /* sigmoid(x . shared_gate_w) (needs shared_inter > 0)  */
  int32_t out_dtype;    /* moe_out_dtype_t of y                                 */
} moe_config_t;

/* Layer weights in checkpoint layout (host memory; read only during create).
 * Matrices are [out, in] row-major; E2M1 codes are packed two per byte with the
 * even input index in the low nibble; block scales run along the input dim.
 *   matrix 0 = gate [I, H], 1 = up [I, H], 2 = down [H, I]
 *   codes[m][e]  : uint8 [rows, K/2]
 *   scales[m][e] : MXFP4 E8M0 uint8 [rows, K/32]; NVFP4 E4M3 uint8 [rows, K/16]
 *   global_scale : NVFP4 only, fp32 [E, 3] per-tensor scale; else NULL
 *   shared_w[m]  : bf16 bit patterns, gate [I_s, H], up [I_s, H], down [H, I_s]
 * The library copies everything during moe_layer_create; the caller may free
 * these buffers when it returns. */
typedef struct {
  const float *router_w;            /* fp32 [E + n_sinks, H]                   */
  const float *router_bias;         /* fp32 [E + n_sinks] added to the logits, */
                                    /* or NULL                                 */
  const uint8_t *const *codes[3];   /* codes[m] -> array of E host pointers    */
  const uint8_t *const *scales[3];  /* scales[m] -> array of E host pointers   */
  const float *global_scale;        /* fp32 [E, 3] or NULL                     */
  const uint16_t *shared_w[3];      /* NULL when shared_inter == 0             */
  const float *shared_gate_w;       /* fp32 [H] when shared_gate, else NULL    */
} moe_weights_t;

/* Optional routing outputs of a forward (all device pointers, each may be
 * NULL).  With NT = E + n_sinks routing targets: logits fp32 [T, NT]; ids
 * int32 [T, k] in descending-logit order (lower index first on ties; ids >= E
 * are sinks); gates fp32 [T, k]; counts int32 [NT]; offsets int32 [NT+1]
 * (exclusive scan of counts); perm int32 [T*k]: sorted position -> pair index
 * p = t*k + j (stable by target, ties by ascending p); inv int32 [T*k]:
 * p -> sorted position. */
typedef struct {
  float *logits;
  int32_t *ids;
  float *gates;
  int32_t *counts;
  int32_t *offsets;
  int32_t *perm;
  int32_t *inv;
} moe_routing_t;

typedef struct {
  uint64_t forwards;       /* forwards run since create                         */
  uint64_t misses;         /* expert copies from the pinned store, cumulative   */
  uint64_t bytes_staged;   /* bytes copied host -> device for misses, cumulative */
  int32_t last_misses;     /* misses of the last forward                        */
  int32_t last_waves;      /* staging waves of the last forward (0 = resident)  */
  int32_t last_active;     /* experts with at least one token, last forward     */
  int32_t last_path;       /* 0 = register-decode kernels (EXACT), 1 = A4      */
                           /* tcgen05 FP4 x FP4, 2 = EXACT on tcgen05 (MXFP4    */
                           /* weights x E4M3 activation pieces), 3 = EXACT on   */
                           /* tcgen05 (NVFP4 / INT4 / FP8 weights decoded into  */
                           /* TMEM x 16-bit activations)                        */
  uint64_t launches;       /* kernels this library launched, cumulative         */
  uint64_t expert_bytes;   /* device-layout bytes of one routed expert          */
  uint64_t device_bytes;   /* HBM held by the layer                             */
  uint64_t pinned_bytes;   /* pinned host memory held by the layer              */
  int32_t device_error;    /* nonzero: a device-side wait gave up (code 1..99   */
                           /* of the first one) or, in the bounds-checked build */
                           /* (libfp4moe_checked.so, -DMOE_DEBUG_CHECKS), an     */
                           /* index read from device data was out of range      */
                           /* (201 target, 202/203 location table, 204 token,   */
                           /* 205 pair); the next moe_forward reports and       */
                           /* clears it                                         */
  int32_t policy;          /* moe_policy_t in force                             */
  uint64_t admitted;       /* staged experts admitted into slots, cumulative    */
  uint64_t prefetched;     /* experts copied into slots by moe_prefetch         */
} moe_stats_t;

/* Memory plan of a configuration without allocating anything (the dry-run
 * placement plan idea of "ro99/strata": --admission-only).  Validates the
 * configuration. */
typedef struct {
  uint64_t expert_bytes;   /* one routed expert in device layout                */
  uint64_t slot_bytes;     /* S resident slots                                  */
  uint64_t staging_bytes;  /* staging ring                                      */
  uint64_t resident_bytes; /* router + shared expert (always in HBM)            */
  uint64_t scratch_bytes;  /* per-forward scratch sized by max_tokens           */
  uint64_t pinned_bytes;   /* pinned host store of all E experts                */
} moe_plan_t;

moe_status_t moe_layer_plan(const moe_config_t *cfg, moe_plan_t *out);

/* Check every block-scale code of the weights against the format (no
 * allocation).  MXFP4: E8M0 codes 0 and 255 are rejected.  NVFP4: E4M3 NaN
 * codes and negative scales are rejected, and the per-tensor scale must be
 * finite and positive.  Returns MOE_ERR_ADMISSION with the expert, matrix and
 * index in moe_last_error(). */
moe_status_t moe_admit(const moe_config_t *cfg, const moe_weights_t *w);

/* Create a layer on cfg->device: admits the scales, copies every routed expert
 * into a pinned host store in device layout, uploads router and shared-expert
 * weights to HBM, allocates S slots, the staging ring and scratch sized by
 * max_tokens.  No expert is resident until moe_set_slot_table.  The stream
 * orders the uploads; the call returns after they complete. */
moe_status_t moe_layer_create(const moe_config_t *cfg, const moe_weights_t *w, void *stream,
                              moe_layer_t *out);

/* Set which experts are resident: slot_of_expert is host int32 [E], each entry
 * a slot index in [0, S) or -1 (kept in host memory).  Rejects out-of-range
 * slots, two experts on one slot and more than S resident experts with
 * MOE_ERR_SLOT_TABLE (the previous table stays in force).  Copies newly
 * resident experts into their slots on `stream`; later forwards on the same
 * stream see the new table.  The table never changes inside moe_forward. */
moe_status_t moe_set_slot_table(moe_layer_t layer, const int32_t *slot_of_expert, void *stream);

/* Who decides which experts are resident (the routing/paging policies
 * none | warm | cache | hybrid of strata.amperor.ai; "Strata, Explained",
 * section 2: an adaptive VRAM cache over every expert pinned in RAM):
 *   STATIC  the caller's slot table, changed only by moe_set_slot_table (a
 *           hottest-first table set once is the "warm" policy); the default;
 *   NONE    no expert is resident: the table is cleared and every expert a
 *           forward needs is staged;
 *   CACHE   the library manages the slots as a cache: after each forward
 *           that staged experts, missed experts are admitted into slots whose
 *           expert that forward did not use (empty slots first, then least
 *           recently used), by a device-to-device copy from the staging
 *           buffer right after the wave that used it; the new table holds for
 *           the next forward;
 *   HYBRID  CACHE on slots [n_pinned, S); the experts in slots [0, n_pinned)
 *           at the time of the call are pinned (a warm fill plus a cache).
 * The current table is the cache's starting content.  Residency never changes
 * what a forward computes: output is bit-identical under every policy.
 * n_pinned is used by HYBRID only (0..S).  Returns after the stream's queued
 * work completes. */
typedef enum { MOE_POLICY_STATIC = 0, MOE_POLICY_NONE = 1, MOE_POLICY_CACHE = 2, MOE_POLICY_HYBRID = 3 } moe_policy_t;
moe_status_t moe_set_policy(moe_layer_t layer, int32_t policy, int32_t n_pinned, void *stream);

/* Prefetch under CACHE or HYBRID: copies the listed experts (host int32
 * [n], a predictor's guess for a coming forward) that are not resident into
 * evictable slots (empty first, then least recently used; experts listed in
 * the same call are not evicted for one another), from the pinned store on the
 * layer's side stream after the work already queued on `stream`; the next
 * forward waits for these copies before its expert passes.  A predictor only
 * reorders work ("ro99/strata", rules list): what the next forward computes
 * does not change.  Experts beyond the evictable slots are skipped.  Other
 * policies: MOE_ERR_INVALID_ARG. */
moe_status_t moe_prefetch(moe_layer_t layer, const int32_t *experts, int32_t n, void *stream);

/* Forward T tokens: x device bf16 [T, H] -> y device [T, H], fp32 or bf16
 * (rounded to nearest even) as the config's out_dtype says.
 * 0 <= T <= max_tokens (T == 0 is a no-op).  x and y must not overlap.
 * When every expert the forward needs is resident, the call only enqueues
 * work on `stream` and returns.  Otherwise it waits for the routing counts
 * (one small device-to-host copy), then copies the missing experts from the
 * pinned store on the layer's side stream, overlapped with compute in waves
 * of at most n_staging experts; it returns once all work is enqueued.  With
 * T <= 128 a layer with a shared expert runs it on a stream of the layer's
 * own, forked from `stream` before the router and joined back before the
 * first kernel that reads its output.
 * dbg (may be NULL) receives the routing tensors of this forward. */
moe_status_t moe_forward(moe_layer_t layer, const void *x, int32_t T, void *y, void *stream,
                         const moe_routing_t *dbg);

/* Same forward from and to HOST memory: copies x (host bf16 [T, H]) to a
 * layer-owned device buffer, runs the forward and copies y back to host
 * [T, H] (fp32 or bf16 per out_dtype).  Returns after y is in host memory. */
moe_status_t moe_forward_host(moe_layer_t layer, const uint16_t *x_host, int32_t T,
                              void *y_host, void *stream);

/* CUDA graph of one forward (launch overhead of a decode step).
 * moe_graph_capture records the forward of T tokens from x (device bf16
 * [T, H]) into y (device [T, H], out_dtype) on `stream` (a created stream, not the
 * legacy default stream) into a CUDA graph without running it; each
 * moe_graph_launch replays it on `stream`, reading the x and writing the y
 * given at capture.  Requires every expert resident (the staged path waits for
 * the routing counts on the host): otherwise MOE_ERR_INVALID_ARG.  A launch
 * after moe_set_slot_table has changed the table returns MOE_ERR_INVALID_ARG.
 * The graph belongs to the caller: moe_graph_destroy before moe_destroy of its
 * layer.  Replays count in moe_stats_t (forwards, launches). */
typedef struct moe_graph *moe_graph_t;
moe_status_t moe_graph_capture(moe_layer_t layer, const void *x, int32_t T, void *y, void *stream,
                               moe_graph_t *out);
moe_status_t moe_graph_launch(moe_graph_t graph, void *stream);
moe_status_t moe_graph_destroy(moe_graph_t graph);

moe_status_t moe_get_stats(moe_layer_t layer, moe_stats_t *out);

/* Per-stage device timing (tracing).  While enabled, every forward records a
 * CUDA event pair around each stage on the stream the stage runs on (the
 * forward's stream, or the layer's own for a forked shared expert, whose
 * time then overlaps the other stages); moe_profile_read
 * waits for those events and returns the accumulated milliseconds and launch
 * counts since the last enable.  Stages: 0 router + top-k, 1 permutation,
 * 2 shared expert, 3 routed gate/up + SwiGLU, 4 routed down + gate scale,
 * 5 combine, 6 waits on staging copies, 7 whole forward, 8 A4 activation
 * quantisation, 9 unused. */
#define MOE_PROFILE_STAGES 10
typedef struct {
  uint64_t forwards;
  double ms[MOE_PROFILE_STAGES];
  uint64_t launches[MOE_PROFILE_STAGES];
} moe_profile_t;

moe_status_t moe_profile_enable(moe_layer_t layer, int32_t enable);
moe_status_t moe_profile_read(moe_layer_t layer, moe_profile_t *out);

/* Routing step alone, for callers that cannot allocate device memory when they
 * call in (a serving loop that plans every byte of HBM once at start-up, or a
 * latency-critical path that must not pay the device-wide synchronisation of
 * cudaMalloc/cudaFree).  The pages have no counterpart of this entry point; it
 * is a library convenience.  Computes, like moe_forward's routing, fp32 logits
 * x * router_w^T (+ router_bias), the top-k expert ids in descending-logit
 * order (lower index first on ties) and the softmax gates renormalised over
 * the k.  Allocates nothing: its scratch (logits and completion counters) is a
 * fixed file-scope device array of 4 MiB + 64 KiB that every GPU loading this
 * library holds until exit.  Limits: T * E <= 2^20, T <= 65536, H a multiple of
 * 4 whose 4-token fp32 tile (16 * H bytes) fits the device's per-block shared
 * memory with the kernel's own (H <= 14524 on a B200, 227 KiB per block),
 * E <= 1024, k <= min(E, 32); router_w must be 16-byte aligned (its rows are
 * read as float4); anything else returns MOE_ERR_INVALID_ARG and launches
 * nothing.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current, so make the
 * first call before any stream capture.  All calls share the array and it
 * keeps the last call's contents (the counters are cleared at every call);
 * calls that overlap on the GPU race on it and must be serialised by the
 * caller.  x: device bf16 [T, H]; router_w: device fp32 [E, H]; router_bias:
 * device fp32 [E] or NULL; ids: device int32 [T, k]; gates: device fp32 [T, k];
 * logits: device fp32 [T, E] or NULL (copied out of the scratch when given). */
moe_status_t moe_route_topk_noalloc(const void *x, int32_t T, int32_t H, const float *router_w,
                                    const float *router_bias, int32_t E, int32_t k, int32_t *ids,
                                    float *gates, float *logits, void *stream);

/* Waits for the layer's work, then frees everything it holds.  NULL is a no-op. */
void moe_destroy(moe_layer_t layer);

/* Thread-local description of the last failure in this thread ("" if none). */
const char *moe_last_error(void);

/* Test hook for host-side failure injection (no GPU fault is ever caused):
 * 1 = the next staging copy reports a failure, 2 = the next device allocation
 * in moe_layer_create fails, 3 = the next forward's device error word is set
 * from the host before its kernels run, so that every bounded device wait of
 * that forward which has to wait gives up (the path a wait takes when its time
 * limit passes; the outputs of that forward are invalid and the following
 * moe_forward reports MOE_ERR_CUDA), 0 = off.  The forward must then return an
 * error status and leave the CUDA context usable. */
moe_status_t moe_debug_inject(moe_layer_t layer, int32_t what);

/* Test hook: synchronously copy up to `bytes` of an internal device buffer of
 * the last forward into host memory.  which: 1 quantised x codes, 2 x scale
 * blocks, 3 h (fp32, A4 path of NVFP4 layers; MXFP4 layers quantise h in the
 * gate/up epilogue and never write it), 4 quantised h codes, 5 h scale blocks, 6 padded
 * row count, 7 padded row -> token, 8 padded row -> pair, 11 O' (fp32);
 * tensor-core EXACT path: 12 x pieces (E4M3, 128-row slot per tile), 13 their
 * scale blocks, 14 h pieces, 15 their scale blocks, 16 tile list, 17 tile
 * count.
 * Returns MOE_ERR_INVALID_ARG for an unknown or absent buffer. */
moe_status_t moe_debug_read(moe_layer_t layer, int32_t which, void *dst_host, uint64_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* MOE_LAYER_H */
