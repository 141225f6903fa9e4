// api.cu -- C ABI and host runtime of the MoE layer: admission, pinned expert
// store in device layout, resident slots, staging ring for misses, forward
// orchestration.
//
// Paging follows the pages' memory hierarchy: every expert pinned in host RAM,
// a budget of hot experts resident on the GPU, the router and shared experts
// always resident ("Strata, Explained", section 2; strata.amperor.ai, the
// "budget ... resident experts/layer" option).  The device layout is packed
// once, at create time, into the pinned store, so a miss costs one plain
// cudaMemcpyAsync ("ro99/strata": a per-staging prepack lands on the
// bottleneck term).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include "moe_internal.h"
#include "tma.cuh"

using namespace moe;

static thread_local std::string g_err;
static int g_inject_create = 0;

static moe_status_t fail(moe_status_t s, const std::string &msg) {
  g_err = msg;
  return s;
}

namespace moe {
// Error text for entry points defined in other translation units.
const char *set_error_text(const std::string &s) {
  g_err = s;
  return g_err.c_str();
}
}  // namespace moe

#define CUDA_TRY(call)                                                                   \
  do {                                                                                   \
    cudaError_t _e = (call);                                                             \
    if (_e != cudaSuccess) {                                                             \
      return fail(MOE_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(_e));     \
    }                                                                                    \
  } while (0)

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

BlobLayout moe::blob_layout(int H, int I, int fmt, int tiled) {
  BlobLayout L{};
  L.fmt = fmt;
  L.tiled = tiled;
  L.G = fmt == MOE_FMT_MXFP4 ? 32 : (fmt == MOE_FMT_NVFP4 ? 16 : 128);
  size_t off = 0;
  for (int m = 0; m < 3; ++m) {
    L.rows[m] = (m < 2) ? I : H;
    L.K[m] = (m < 2) ? H : I;
    L.codes[m] = off;
    const size_t cb = fmt == MOE_FMT_FP8B128 ? (size_t)L.rows[m] * L.K[m] : (size_t)L.rows[m] * L.K[m] / 2;
    off = align256(off + cb);
  }
  for (int m = 0; m < 3; ++m) {
    L.scales[m] = off;
    size_t sb = (size_t)L.rows[m] * L.K[m] / L.G;                                  // one byte per block
    if (fmt == MOE_FMT_INT4G128) sb *= 2;                                           // bf16 per row and group
    if (fmt == MOE_FMT_FP8B128) sb = (size_t)(L.rows[m] / 128) * (L.K[m] / 128) * 4;  // fp32 per 128 x 128
    off = align256(off + sb);
  }
  for (int m = 0; m < 3; ++m) L.sref[m] = 0;
  L.glob = 0;
  if (fmt == MOE_FMT_MXFP4) {
    for (int m = 0; m < 3; ++m) {
      L.sref[m] = off;
      off = align256(off + (size_t)L.rows[m]);
    }
  } else if (fmt == MOE_FMT_NVFP4) {
    L.glob = off;
    off = align256(off + 3 * sizeof(float));
  }
  L.bytes = off;
  return L;
}

struct moe_layer {
  moe_config_t cfg{};
  BlobLayout L{};
  int wf = 0;
  int n_staging = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_copied[2] = {}, ev_done[2] = {}, ev_counts = nullptr, ev_fwd_done = nullptr;
  // decode-sized batches run the shared expert on its own stream, forked
  // before the router and joined before the first kernel that reads its output
  cudaStream_t sh_stream = nullptr;
  cudaEvent_t ev_sh_fork = nullptr, ev_sh_join = nullptr;
  bool sh_join_pending = false;
  // device memory
  std::vector<void *> dev;
  float *router_w = nullptr, *router_b = nullptr;
  float *router_parts = nullptr;     // split-K partial logits of the prefill router GEMM
  uint16_t *shared_w[3] = {};
  uint8_t *slots = nullptr, *staging = nullptr;
  int *loc_resident = nullptr, *loc_pass = nullptr;
  CodeMaps maps{};
  int *h_err = nullptr;                      // mapped pinned error word, read by the host
  int *d_err = nullptr;                      // device error word (ErrWord) the kernels poll and write
  float *logits = nullptr, *gates = nullptr;
  int *ids = nullptr, *counts = nullptr, *offsets = nullptr, *perm = nullptr, *inv = nullptr;
  TileInfo *tiles = nullptr;
  int *n_tiles = nullptr, *active = nullptr, *prow_token = nullptr, *prow_pair = nullptr;
  uint16_t *xf16 = nullptr, *hbuf = nullptr, *sh_h = nullptr, *xin = nullptr;
  // shared expert on the tensor core (prefill): bf16 weight maps and the h map
  CUtensorMap sh_map[3];
  CUtensorMap sh_hmap;
  float *xs = nullptr, *hscale = nullptr, *oprime = nullptr, *sh_s = nullptr, *yout = nullptr;
  int *router_counter = nullptr, *tiles_done = nullptr, *comb_cnt = nullptr;
  // A4 (activation FP4) path
  bool a4 = false;
  size_t a4_rows = 0;
  A4Maps a4maps{};
  uint8_t *xq = nullptr, *xsf = nullptr, *hq = nullptr, *hsf = nullptr;
  float *xG = nullptr, *hG = nullptr, *h32 = nullptr;
  int *n_prows = nullptr;
  uint16_t *xg = nullptr;            // dequantising path: x rows in padded expert order
  float *xgs = nullptr;              // their f16 scales (NVFP4)
  int *a4_work = nullptr;            // [kWorkCtrs] item counters of the two A4 passes
  // EXACT numerics of MXFP4 experts on the tensor core (E4M3 activation pieces)
  bool tc = false;
  int n_sms = 148;
  size_t tc_rows = 0;
  TcMaps tcmaps{};
  uint8_t *txq = nullptr, *txsf = nullptr, *thq = nullptr, *thsf = nullptr;
  int *tc_work = nullptr;            // [kWorkCtrs] item counters of the expert passes
  int *tile_done = nullptr;          // [tc tiles] gate/up items finished per tile (decode hand-over)
  CUtensorMap tc_act[2];             // activation-piece maps of the two passes (x pieces, h pieces)
  // EXACT numerics of NVFP4 experts at prefill sizes on the tensor core
  // (weights decoded to bf16 in shared memory)
  bool nv = false;
  DqMaps dqmaps{};
  int *dq_work = nullptr;            // [kWorkCtrs] item counters of the two passes
  int cur_T = 0;                     // tokens of the forward being enqueued
  // host
  uint8_t *store = nullptr;          // pinned: E x blob bytes
  int *h_counts = nullptr;           // pinned [E]
  int *h_loc = nullptr;              // pinned [E]
  std::vector<int> slot_of;
  int n_resident = 0;
  uint64_t table_version = 0;        // bumped by every change of the slot table
  size_t max_prows = 0, max_tiles = 0;
  // library-managed residency (moe_set_policy): the slot holding each
  // expert changes only between forwards, by admission of staged misses
  // (cache / hybrid) or by moe_prefetch
  int policy = MOE_POLICY_STATIC;
  int n_pinned = 0;                  // hybrid: slots [0, n_pinned) are never evicted
  std::vector<int> expert_of_slot;   // [S] expert in each slot, -1 = empty
  std::vector<uint64_t> last_use;    // [E] forward index of each expert's last use
  cudaEvent_t ev_prefetch = nullptr; // prefetch copies done (side stream)
  bool prefetch_pending = false;
  moe_stats_t st{};
  int inject = 0;
  bool staging_used = false;
  // tracing: CUDA event pairs per stage, read back by moe_profile_read
  struct Pending {
    int stage;
    cudaEvent_t a, b;
  };
  bool prof = false;
  std::vector<Pending> pend;
  std::vector<cudaEvent_t> evpool;
  moe_profile_t prof_acc{};
};

static cudaEvent_t take_event(moe_layer *L) {
  if (!L->evpool.empty()) {
    cudaEvent_t e = L->evpool.back();
    L->evpool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return e;
}

// Records an event pair around one stage of a forward when tracing is on, and
// counts the stage's kernel launches.
struct StageTimer {
  moe_layer *L;
  int stage;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  StageTimer(moe_layer *L_, int st, cudaStream_t s_) : L(L_), stage(st), s(s_) {
    if (L->prof && (a = take_event(L))) cudaEventRecord(a, s);
  }
  void launched(int n) {
    L->st.launches += n;
    L->prof_acc.launches[stage] += n;
  }
  void end() {
    if (!a) return;
    cudaEvent_t b = take_event(L);
    if (!b) {
      L->evpool.push_back(a);
      a = nullptr;
      return;
    }
    cudaEventRecord(b, s);
    L->pend.push_back({stage, a, b});
    a = nullptr;
  }
};

// ------------------------------------------------------------------ helpers
static moe_status_t check_config(const moe_config_t *c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
  if (c->hidden <= 0 || c->hidden % 256) return fail(MOE_ERR_INVALID_ARG, "hidden must be a positive multiple of 256");
  if (c->inter <= 0 || c->inter % 128) return fail(MOE_ERR_INVALID_ARG, "inter must be a positive multiple of 128");
  if (c->n_experts < 1 || c->n_experts > kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "n_experts must be in 1..1024");
  if (c->n_sinks < 0 || c->shared_gate < 0 || c->shared_gate > 1 ||
      c->n_experts + c->n_sinks + c->shared_gate > kMaxExperts)
    return fail(MOE_ERR_INVALID_ARG, "need n_sinks >= 0, shared_gate 0 or 1, n_experts + n_sinks + shared_gate <= 1024");
  if (c->top_k < 1 || c->top_k > std::min(c->n_experts + c->n_sinks, kMaxTopK))
    return fail(MOE_ERR_INVALID_ARG, "top_k must be in 1..min(n_experts + n_sinks, 32)");
  if (c->shared_inter < 0 || c->shared_inter % 128) return fail(MOE_ERR_INVALID_ARG, "shared_inter must be 0 or a multiple of 128");
  if (c->shared_gate && c->shared_inter == 0) return fail(MOE_ERR_INVALID_ARG, "shared_gate needs a shared expert");
  if (c->fmt < MOE_FMT_MXFP4 || c->fmt > MOE_FMT_FP8B128)
    return fail(MOE_ERR_INVALID_ARG, "fmt must be MXFP4, NVFP4, INT4G128 or FP8B128");
  if (c->renormalize != 0 && c->renormalize != 1) return fail(MOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (c->scoring != MOE_SCORING_SOFTMAX && c->scoring != MOE_SCORING_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "scoring must be SOFTMAX or SIGMOID");
  if (c->out_dtype != MOE_OUT_F32 && c->out_dtype != MOE_OUT_BF16) return fail(MOE_ERR_INVALID_ARG, "out_dtype must be F32 or BF16");
  if (c->numerics != MOE_NUMERICS_EXACT && c->numerics != MOE_NUMERICS_A4)
    return fail(MOE_ERR_INVALID_ARG, "numerics must be EXACT or A4");
  if (c->numerics == MOE_NUMERICS_A4 && c->fmt != MOE_FMT_MXFP4 && c->fmt != MOE_FMT_NVFP4)
    return fail(MOE_ERR_UNSUPPORTED, "A4 numerics quantises activations to the experts' FP4 format: "
                                     "MXFP4 and NVFP4 layers only");
  if (c->n_slots < 0 || c->n_slots > c->n_experts) return fail(MOE_ERR_INVALID_ARG, "n_slots must be in 0..n_experts");
  if (c->max_tokens < 1 || (int64_t)c->max_tokens * c->top_k > (1 << 30))
    return fail(MOE_ERR_INVALID_ARG, "max_tokens must be >= 1 and max_tokens * top_k <= 2^30");
  if (c->n_staging < 0 || c->n_staging > 2 * kPtrListMax) return fail(MOE_ERR_INVALID_ARG, "n_staging must be in 0..512");
  if (c->n_slots < c->n_experts && c->n_staging == 1) return fail(MOE_ERR_INVALID_ARG, "n_staging must be >= 2 when n_slots < n_experts");
  return MOE_OK;
}

static int default_staging(const moe_config_t *c) {
  if (c->n_slots >= c->n_experts) return 0;
  if (c->n_staging > 0) return c->n_staging;
  return std::max(2, std::min(c->n_experts - c->n_slots, 64));
}

// Routing targets (experts, then sinks) and router logit rows (targets, then
// the shared-expert gate row when the layer has one).
static int n_targets(const moe_config_t *c) { return c->n_experts + c->n_sinks; }
static int n_logit_rows(const moe_config_t *c) { return n_targets(c) + c->shared_gate; }

struct Sizes {
  size_t P, max_prows, max_tiles, a4_rows, tc_tiles;
};
static Sizes sizes_of(const moe_config_t *c) {
  Sizes s;
  s.P = (size_t)c->max_tokens * c->top_k;
  const size_t act = std::min<size_t>(c->n_experts, s.P);
  s.max_prows = s.P + 8 * act;
  s.max_tiles = s.P / 8 + act + 1;
  s.a4_rows = s.P + 128 * act + 128;     // padded to 128 rows per expert, + one tile of slack
  // tensor-core EXACT path: tiles of 8 tokens only while P <= 12 * active experts
  // (then at most 2.5 x act tiles), else tiles of 56 tokens
  s.tc_tiles = std::max(s.P / 56 + act, (5 * act) / 2 + 1) + 2;
  return s;
}

static size_t a4_scratch_bytes(const moe_config_t *c) {
  if (c->numerics != MOE_NUMERICS_A4) return 0;
  const Sizes z = sizes_of(c);
  const size_t H = c->hidden, I = c->inter, G = c->fmt == MOE_FMT_MXFP4 ? 32 : 16;
  size_t b = align256(z.a4_rows * H / 2) + align256(z.a4_rows * H / G) + align256(z.a4_rows * 4);
  b += align256(z.a4_rows * I * 4) + align256(z.a4_rows * I / 2) + align256(z.a4_rows * I / G) + align256(z.a4_rows * 4);
  b += align256(z.P * H * 4) + align256(4) + align256(kWorkCtrs * sizeof(int));
  return b;
}

static bool uses_tc(const moe_config_t *c) {
  return c->numerics == MOE_NUMERICS_EXACT && c->fmt == MOE_FMT_MXFP4;
}

// Blob layout of a layer's experts: tile-major for the tensor-core EXACT path,
// gate/up interleaved per 64 rows for A4, checkpoint order otherwise.
static int blob_tiling(const moe_config_t *c) {
  return uses_tc(c) ? 1 : (c->numerics == MOE_NUMERICS_A4 ? 2 : 0);
}

// NVFP4 layers in EXACT numerics: prefill-sized batches run the tensor-core
// kernels that decode weights to bf16 in shared memory (decode-sized batches
// keep the register-decode kernels); both read the same blob layout.
static bool uses_dq(const moe_config_t *c) {
  return c->numerics == MOE_NUMERICS_EXACT && c->fmt != MOE_FMT_MXFP4;
}
// INT4 group-128 and FP8 block-128 experts run only on the dequantising
// tensor-core kernels (every batch size)
static bool dq_only(const moe_config_t *c) { return c->fmt == MOE_FMT_INT4G128 || c->fmt == MOE_FMT_FP8B128; }

static size_t tc_scratch_bytes(const moe_config_t *c) {
  if (uses_dq(c)) {
    const Sizes z = sizes_of(c);
    return align256(kWorkCtrs * sizeof(int)) + align256(z.max_prows * c->hidden * 2) + align256(z.max_prows * 4) +
           align256(4);
  }
  if (!uses_tc(c)) return 0;
  const Sizes z = sizes_of(c);
  const size_t R = z.tc_tiles * kTcSlotRows, H = c->hidden, I = c->inter;
  return align256(R * H) + align256(R * H / 32) + align256(R * I) + align256(R * I / 32) +
         align256(kWorkCtrs * sizeof(int)) + align256(z.tc_tiles * sizeof(int));
}

static size_t scratch_bytes(const moe_config_t *c) {
  const Sizes z = sizes_of(c);
  const size_t T = c->max_tokens, H = c->hidden, I = c->inter, Is = c->shared_inter;
  size_t b = 0;
  const size_t NT = n_targets(c), NR = n_logit_rows(c);
  b += align256(T * NR * 4) + align256(z.P * 4) * 4 + align256(NT * 4) + align256((NT + 1) * 4);
  b += align256(z.max_tiles * sizeof(TileInfo)) + 2 * align256(4) + 2 * align256(z.max_prows * 4);
  b += align256(T * H * 2) + align256(T * (H / kChunk) * 4);
  b += align256(z.max_prows * I * 2) + align256(z.max_prows * (I / kChunk) * 4);
  b += align256(z.P * H * 4);
  if (Is) b += align256(T * Is * 2) + align256(T * H * 4);
  b += align256(((T + 3) / 4) * 4) + align256(4) + align256(T * (H / 128) * 4);
  b += align256(T * H * 2) + align256(T * H * 4);
    if (T >= 256) b += align256((size_t)(4 << 20) * 4);     // split-K partial logits (prefill router)
  return b;
}

template <typename P>
static moe_status_t dalloc(moe_layer *L, P **p, size_t bytes) {
  if (g_inject_create == 2) {
    g_inject_create = 0;
    return fail(MOE_ERR_OOM, "injected device allocation failure");
  }
  void *q = nullptr;
  cudaError_t e = cudaMalloc(&q, std::max<size_t>(bytes, 256));
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(MOE_ERR_OOM, std::string("cudaMalloc failed: ") + cudaGetErrorString(e));
  }
  L->dev.push_back(q);
  *p = reinterpret_cast<P *>(q);
  return MOE_OK;
}

#define ST_TRY(x)                 \
  do {                            \
    moe_status_t _s = (x);        \
    if (_s != MOE_OK) return _s;  \
  } while (0)

static void free_layer(moe_layer *L) {
  if (!L) return;
  cudaSetDevice(L->cfg.device);
  cudaDeviceSynchronize();
  for (void *p : L->dev) cudaFree(p);
  if (L->store) cudaFreeHost(L->store);
  if (L->h_counts) cudaFreeHost(L->h_counts);
  if (L->h_err) cudaFreeHost(L->h_err);
  if (L->h_loc) cudaFreeHost(L->h_loc);
  for (int i = 0; i < 2; ++i) {
    if (L->ev_copied[i]) cudaEventDestroy(L->ev_copied[i]);
    if (L->ev_done[i]) cudaEventDestroy(L->ev_done[i]);
  }
  if (L->ev_counts) cudaEventDestroy(L->ev_counts);
  if (L->ev_fwd_done) cudaEventDestroy(L->ev_fwd_done);
  if (L->ev_prefetch) cudaEventDestroy(L->ev_prefetch);
  for (auto &p : L->pend) { cudaEventDestroy(p.a); cudaEventDestroy(p.b); }
  for (auto e : L->evpool) cudaEventDestroy(e);
  if (L->ev_sh_fork) cudaEventDestroy(L->ev_sh_fork);
  if (L->ev_sh_join) cudaEventDestroy(L->ev_sh_join);
  if (L->side) cudaStreamDestroy(L->side);
  if (L->sh_stream) cudaStreamDestroy(L->sh_stream);
  delete L;
}

// ------------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over the code bytes of matrix m of every blob in a region:
// (K/2 bytes, rows, blob index), box box_bytes x box_rows x 1, no swizzle.
static moe_status_t make_code_map(CUtensorMap *map, const uint8_t *region, int nblobs, const BlobLayout &L, int m,
                                  int box_rows, int box_bytes = 64) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t row_bytes = L.fmt == MOE_FMT_FP8B128 ? (cuuint64_t)L.K[m] : (cuuint64_t)(L.K[m] / 2);
  cuuint64_t dims[3] = {row_bytes, (cuuint64_t)L.rows[m], (cuuint64_t)nblobs};
  cuuint64_t strides[2] = {row_bytes, (cuuint64_t)L.bytes};
  cuuint32_t box[3] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void *)(region + L.codes[m]), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d) for matrix %d", (int)r, m);
    return fail(MOE_ERR_CUDA, buf);
  }
  return MOE_OK;
}

// A4 weight map: (K/2 bytes, rows, blob index), box 128 bytes x 128 rows, 128-byte swizzle.
static moe_status_t make_a4_weight_map(CUtensorMap *map, const uint8_t *region, int nblobs, const BlobLayout &L,
                                       int m) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  // gate/up of the interleaved layout: one matrix of 2I rows from codes[0]
  const cuuint64_t rows = (L.tiled == 2 && m == 0) ? (cuuint64_t)(2 * L.rows[0]) : (cuuint64_t)L.rows[m];
  cuuint64_t dims[3] = {(cuuint64_t)(L.K[m] / 2), rows, (cuuint64_t)nblobs};
  cuuint64_t strides[2] = {(cuuint64_t)(L.K[m] / 2), (cuuint64_t)L.bytes};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void *)(region + L.codes[m]), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for an A4 weight map");
  return MOE_OK;
}

// A4 activation map: (row bytes, rows), box 128 bytes x 128 rows, 128-byte swizzle.
static moe_status_t make_a4_act_map(CUtensorMap *map, const uint8_t *base, size_t row_bytes, size_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for an A4 activation map");
  return MOE_OK;
}

// Tensor-core EXACT weight map over a tiled code region: 4-D (128 elements,
// 256 rows of 64 bytes, chunk, blob), box 128 x 256 x 1 x 1 = one contiguous
// 16 KB chunk, unpacked by the TMA to one byte per element (8 code bytes + 8
// empty bytes per 16 elements, the shared-memory form the f8f6f4 MMA kinds
// read), 128-byte swizzle.
static moe_status_t make_tc_weight_map(CUtensorMap *map, const uint8_t *region, int nblobs, const BlobLayout &L,
                                       bool gate_up) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int H = L.K[0], I = L.rows[0];
  const size_t nchunks = gate_up ? (size_t)(I / 128) * (H / 128) : (size_t)(H / 256) * (I / 128);
  cuuint64_t dims[4] = {128, 256, (cuuint64_t)nchunks, (cuuint64_t)nblobs};
  cuuint64_t strides[3] = {64, (cuuint64_t)kTcChunk, (cuuint64_t)L.bytes};
  cuuint32_t box[4] = {128, 256, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 4, (void *)(region + L.codes[gate_up ? 0 : 2]), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d) for a tiled weight map", (int)r);
    return fail(MOE_ERR_CUDA, buf);
  }
  return MOE_OK;
}

// Activation-piece rows [rows, row_bytes] E4M3: box 128 bytes x 16 rows, 128-byte swizzle.
static moe_status_t make_piece_map(CUtensorMap *map, const void *base, size_t row_bytes, size_t rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128, 16};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for an activation-piece map");
  return MOE_OK;
}

// bf16 row-major [rows, K] map, box 64 elements (128 B) x box_rows rows, 128-byte swizzle.
static moe_status_t make_bf16_map(CUtensorMap *map, const void *base, size_t K, size_t rows, int box_rows = 128) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for a bf16 map");
  return MOE_OK;
}

// Tokens from which the shared expert runs on the tensor core (below that the
// register kernels, which split K over a cluster, keep more SMs busy).
constexpr int kDenseTcMinTokens = 256;
constexpr size_t kRouterPartFloats = (size_t)4 << 20;   // 16 MiB of split-K partial logits

// ------------------------------------------------------------------ residency policies
// Slots a CACHE / HYBRID layer may overwrite now: not pinned, and either empty
// or holding an expert that `busy` does not mark; empty first, then least
// recently used (ties: lower slot).
static std::vector<int> evictable_slots(const moe_layer *L, const std::vector<char> &busy) {
  std::vector<int> cand;
  const int S = L->cfg.n_slots;
  const int first = L->policy == MOE_POLICY_HYBRID ? L->n_pinned : 0;
  for (int v = first; v < S; ++v) {
    const int u = L->expert_of_slot[v];
    if (u < 0 || !busy[u]) cand.push_back(v);
  }
  std::stable_sort(cand.begin(), cand.end(), [&](int a, int b) {
    const int ua = L->expert_of_slot[a], ub = L->expert_of_slot[b];
    const uint64_t ka = ua < 0 ? 0 : L->last_use[ua] + 1, kb = ub < 0 ? 0 : L->last_use[ub] + 1;
    return ka < kb;
  });
  return cand;
}

// Admission plan of one staged forward (CACHE / HYBRID): slot for each miss
// (index into `misses`) or -1.  Misses with more tokens are admitted first;
// only slots whose expert this forward does not use are taken.
static std::vector<int> plan_admission(const moe_layer *L, const std::vector<int> &misses) {
  std::vector<int> slot(misses.size(), -1);
  if (L->policy != MOE_POLICY_CACHE && L->policy != MOE_POLICY_HYBRID) return slot;
  const int E = L->cfg.n_experts;
  std::vector<char> busy(E, 0);
  for (int e = 0; e < E; ++e) busy[e] = L->h_counts[e] > 0;
  const std::vector<int> cand = evictable_slots(L, busy);
  std::vector<int> order(misses.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = (int)i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return L->h_counts[misses[a]] > L->h_counts[misses[b]]; });
  for (size_t i = 0; i < order.size() && i < cand.size(); ++i) slot[order[i]] = cand[i];
  return slot;
}

// Bring the device copies of the slot table up to date with the host's
// (slot_of), ordered on `s` behind the work already queued there.  The sources
// are pageable, so the call returns once they have been read.
static moe_status_t push_table(moe_layer *L, cudaStream_t s) {
  const int E = L->cfg.n_experts;
  std::vector<int> loc(E);
  int n = 0;
  for (int e = 0; e < E; ++e) {
    const int v = L->slot_of[e];
    loc[e] = v >= 0 ? v : kLocAbsent;
    n += v >= 0;
  }
  CUDA_TRY(cudaMemcpyAsync(L->loc_resident, loc.data(), sizeof(int) * E, cudaMemcpyHostToDevice, s));
  L->n_resident = n;
  L->table_version += 1;
  return MOE_OK;
}

// An earlier forward's kernels recorded an error: report it and clear both
// words (the device word on the caller's stream, finished before returning,
// so that the next forward starts clean on any stream).
static moe_status_t report_device_error(moe_layer *L, void *stream) {
  char buf[128];
  snprintf(buf, sizeof buf, "a device-side wait or check of an earlier forward gave up (code %d); outputs of that "
           "forward are invalid", *(volatile int *)L->h_err);
  *(volatile int *)L->h_err = 0;
  cudaSetDevice(L->cfg.device);
  if (cudaMemsetAsync(L->d_err, 0, sizeof(int), (cudaStream_t)stream) != cudaSuccess ||
      cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    (void)cudaGetLastError();
  return fail(MOE_ERR_CUDA, buf);
}

// ------------------------------------------------------------------ C ABI
extern "C" {

const char *moe_last_error(void) { return g_err.c_str(); }

moe_status_t moe_layer_plan(const moe_config_t *cfg, moe_plan_t *out) {
  ST_TRY(check_config(cfg));
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  const BlobLayout L = blob_layout(cfg->hidden, cfg->inter, cfg->fmt, blob_tiling(cfg));
  out->expert_bytes = L.bytes;
  out->slot_bytes = (uint64_t)L.bytes * cfg->n_slots;
  out->staging_bytes = (uint64_t)L.bytes * default_staging(cfg);
  out->resident_bytes = (uint64_t)n_logit_rows(cfg) * cfg->hidden * 4 + n_logit_rows(cfg) * 4 +
                        (uint64_t)3 * cfg->shared_inter * cfg->hidden * 2;
  out->scratch_bytes = scratch_bytes(cfg) + a4_scratch_bytes(cfg) + tc_scratch_bytes(cfg);
  out->pinned_bytes = (uint64_t)L.bytes * cfg->n_experts;
  return MOE_OK;
}

moe_status_t moe_admit(const moe_config_t *cfg, const moe_weights_t *w) {
  ST_TRY(check_config(cfg));
  if (!w || !w->router_w) return fail(MOE_ERR_INVALID_ARG, "weights or router_w is NULL");
  const BlobLayout L = blob_layout(cfg->hidden, cfg->inter, cfg->fmt, 0);
  for (int m = 0; m < 3; ++m)
    if (!w->codes[m] || !w->scales[m]) return fail(MOE_ERR_INVALID_ARG, "codes/scales table is NULL");
  if (cfg->shared_inter > 0 && (!w->shared_w[0] || !w->shared_w[1] || !w->shared_w[2]))
    return fail(MOE_ERR_INVALID_ARG, "shared expert weights are NULL");
  if (cfg->fmt == MOE_FMT_NVFP4 && !w->global_scale)
    return fail(MOE_ERR_INVALID_ARG, "NVFP4 needs global_scale [E,3]");
  if (cfg->shared_gate && !w->shared_gate_w)
    return fail(MOE_ERR_INVALID_ARG, "shared_gate needs shared_gate_w [H]");
  for (int e = 0; e < cfg->n_experts; ++e) {
    for (int m = 0; m < 3; ++m) {
      const uint8_t *s = w->scales[m][e];
      if (!s || !w->codes[m][e]) return fail(MOE_ERR_INVALID_ARG, "NULL expert pointer");
      if (cfg->fmt == MOE_FMT_INT4G128 || cfg->fmt == MOE_FMT_FP8B128) {
        // INT4: bf16 scales [rows, K/128], NaN / infinity rejected; FP8: fp32
        // inverse scales [rows/128, K/128] must be finite and positive, and an
        // E4M3 NaN code (S.1111.111) in the weights is rejected
        const bool i4 = cfg->fmt == MOE_FMT_INT4G128;
        const size_t n = i4 ? (size_t)L.rows[m] * (L.K[m] / 128) : (size_t)(L.rows[m] / 128) * (L.K[m] / 128);
        for (size_t i = 0; i < n; ++i) {
          bool bad;
          if (i4) {
            uint16_t b;
            memcpy(&b, s + 2 * i, 2);
            bad = (b & 0x7F80u) == 0x7F80u;
          } else {
            float f;
            memcpy(&f, s + 4 * i, 4);
            bad = !(f > 0.0f) || f == INFINITY;
          }
          if (bad) {
            char buf[160];
            snprintf(buf, sizeof buf, "scale admission failed: expert %d matrix %d index %zu", e, m, i);
            return fail(MOE_ERR_ADMISSION, buf);
          }
        }
        if (!i4) {
          const uint8_t *q = w->codes[m][e];
          const size_t nq = (size_t)L.rows[m] * L.K[m];
          for (size_t i = 0; i < nq; ++i)
            if ((q[i] & 0x7Fu) == 0x7Fu) {
              char buf[160];
              snprintf(buf, sizeof buf, "weight admission failed: E4M3 NaN code in expert %d matrix %d index %zu", e, m, i);
              return fail(MOE_ERR_ADMISSION, buf);
            }
        }
        continue;
      }
      const size_t n = (size_t)L.rows[m] * L.K[m] / L.G;
      for (size_t i = 0; i < n; ++i) {
        const unsigned c = s[i];
        const bool bad = cfg->fmt == MOE_FMT_MXFP4 ? (c == 0u || c == 255u)
                                                   : ((c & 0x7Fu) == 0x7Fu || (c & 0x80u));
        if (bad) {
          char buf[160];
          snprintf(buf, sizeof buf, "scale admission failed: expert %d matrix %d index %zu code %u", e, m, i, c);
          return fail(MOE_ERR_ADMISSION, buf);
        }
      }
      if (cfg->fmt == MOE_FMT_NVFP4) {
        const float gsc = w->global_scale[e * 3 + m];
        if (!(gsc > 0.0f) || gsc == INFINITY) {
          char buf[128];
          snprintf(buf, sizeof buf, "scale admission failed: per-tensor scale of expert %d matrix %d", e, m);
          return fail(MOE_ERR_ADMISSION, buf);
        }
      }
    }
  }
  return MOE_OK;
}

// Tile-major codes and scales (layout tiled = 1).
static void pack_expert_tiled(const BlobLayout &L, const moe_weights_t *w, int e, uint8_t *dst) {
  const int H = L.K[0], I = L.rows[0];
  const int ns_gu = H / 128, ns_dn = I / 128;
  // gate / up: chunk (rb, slab) = [gate 128 rows][up 128 rows] x 64 bytes
  for (int rb = 0; rb < I / 128; ++rb)
    for (int slab = 0; slab < ns_gu; ++slab)
      for (int mat = 0; mat < 2; ++mat) {
        const size_t chunk = (size_t)rb * ns_gu + slab;
        uint8_t *cd = dst + L.codes[0] + chunk * kTcChunk + (size_t)mat * (kTcChunk / 2);
        uint8_t *sd = dst + L.scales[0] + chunk * kTcSfChunk + (size_t)mat * 512;
        const uint8_t *cs = w->codes[mat][e], *ss = w->scales[mat][e];
        for (int r = 0; r < 128; ++r) {
          const size_t row = (size_t)rb * 128 + r;
          memcpy(cd + r * 64, cs + row * (H / 2) + (size_t)slab * 64, 64);
          for (int c = 0; c < 4; ++c) sd[sf_offset(4, r, c)] = ss[row * (H / 32) + slab * 4 + c];
        }
      }
  // down: chunk (rb, slab) = 256 rows x 64 bytes; scale halves rows 0..127, 128..255
  for (int rb = 0; rb < H / 256; ++rb)
    for (int slab = 0; slab < ns_dn; ++slab) {
      const size_t chunk = (size_t)rb * ns_dn + slab;
      uint8_t *cd = dst + L.codes[2] + chunk * kTcChunk;
      uint8_t *sd = dst + L.scales[2] + chunk * kTcSfChunk;
      const uint8_t *cs = w->codes[2][e], *ss = w->scales[2][e];
      for (int r = 0; r < 256; ++r) {
        const size_t row = (size_t)rb * 256 + r;
        memcpy(cd + r * 64, cs + row * (I / 2) + (size_t)slab * 64, 64);
        for (int c = 0; c < 4; ++c) sd[(r / 128) * 512 + sf_offset(4, r % 128, c)] = ss[row * (I / 32) + slab * 4 + c];
      }
    }
}

// Row c of the interleaved gate/up matrix (layout tiled = 2): matrix (c / 64) % 2
// (0 gate, 1 up), row (c / 128) * 64 + c % 64 of it.
static void a4_gu_source(int c, int *mat, int *row) {
  *mat = (c >> 6) & 1;
  *row = (c >> 7) * 64 + (c & 63);
}

static void pack_expert(const moe_config_t *cfg, const BlobLayout &L, const moe_weights_t *w, int e,
                        uint8_t *dst) {
  if (L.tiled == 1) {
    pack_expert_tiled(L, w, e, dst);
    return;
  }
  if (cfg->fmt == MOE_FMT_INT4G128 || cfg->fmt == MOE_FMT_FP8B128) {
    for (int m = 0; m < 3; ++m) {
      const int rows = L.rows[m], K = L.K[m];
      if (cfg->fmt == MOE_FMT_FP8B128) {
        // codes and the [rows/128, K/128] fp32 block scales as they are
        memcpy(dst + L.codes[m], w->codes[m][e], (size_t)rows * K);
        memcpy(dst + L.scales[m], w->scales[m][e], (size_t)(rows / 128) * (K / 128) * 4);
      } else {
        // codes as they are; the bf16 scales of each (128-row block, K group)
        // contiguous (256 bytes), so that one slab's scales are one copy
        memcpy(dst + L.codes[m], w->codes[m][e], (size_t)rows * K / 2);
        const int ng = K / 128;
        const uint8_t *src = w->scales[m][e];
        for (int r = 0; r < rows; ++r)
          for (int g = 0; g < ng; ++g)
            memcpy(dst + L.scales[m] + ((size_t)(r / 128) * ng + g) * 256 + (r % 128) * 2,
                   src + ((size_t)r * ng + g) * 2, 2);
      }
    }
    return;
  }
  if (L.tiled == 2) {
    // gate and up interleaved per 64 rows into one matrix of 2I rows
    const int H = L.K[0], I = L.rows[0], nsf = H / L.G;
    for (int c = 0; c < 2 * I; ++c) {
      int mat, row;
      a4_gu_source(c, &mat, &row);
      memcpy(dst + L.codes[0] + (size_t)c * (H / 2), w->codes[mat][e] + (size_t)row * (H / 2), (size_t)H / 2);
      const uint8_t *src = w->scales[mat][e] + (size_t)row * nsf;
      for (int col = 0; col < nsf; ++col) dst[L.scales[0] + sf_offset(nsf, c, col)] = src[col];
    }
  }
  for (int m = L.tiled == 2 ? 2 : 0; m < 3; ++m) {
    const size_t ncode = (size_t)L.rows[m] * L.K[m] / 2;
    const size_t nsc = (size_t)L.rows[m] * L.K[m] / L.G;
    memcpy(dst + L.codes[m], w->codes[m][e], ncode);
    {
      const int nsf = L.K[m] / L.G;
      const uint8_t *src = w->scales[m][e];
      for (int r = 0; r < L.rows[m]; ++r)
        for (int c = 0; c < nsf; ++c) dst[L.scales[m] + sf_offset(nsf, r, c)] = src[(size_t)r * nsf + c];
    }
    (void)nsc;
    if (cfg->fmt == MOE_FMT_MXFP4) {
      const int per = L.K[m] / L.G;
      const uint8_t *s = w->scales[m][e];
      for (int r = 0; r < L.rows[m]; ++r) {
        uint8_t mx = 1;
        for (int i = 0; i < per; ++i) mx = std::max(mx, s[(size_t)r * per + i]);
        dst[L.sref[m] + r] = mx;
      }
    }
  }
  if (cfg->fmt == MOE_FMT_NVFP4) {
    float g[3] = {w->global_scale[e * 3 + 0], w->global_scale[e * 3 + 1], w->global_scale[e * 3 + 2]};
    memcpy(dst + L.glob, g, sizeof g);
  }
}

moe_status_t moe_layer_create(const moe_config_t *cfg, const moe_weights_t *w, void *stream,
                              moe_layer_t *out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  ST_TRY(moe_admit(cfg, w));
  CUDA_TRY(cudaSetDevice(cfg->device));
  cudaStream_t s = (cudaStream_t)stream;
  moe_layer *L = new moe_layer();
  L->cfg = *cfg;
  L->L = blob_layout(cfg->hidden, cfg->inter, cfg->fmt, blob_tiling(cfg));
  L->wf = cfg->fmt == MOE_FMT_MXFP4 ? WF_MX : (cfg->fmt == MOE_FMT_NVFP4 ? WF_NV : -1);
  L->n_staging = default_staging(cfg);
  L->cfg.n_staging = L->n_staging;
  const int E = cfg->n_experts, H = cfg->hidden, I = cfg->inter, Is = cfg->shared_inter;
  const Sizes z = sizes_of(cfg);
  L->max_prows = z.max_prows;
  L->max_tiles = z.max_tiles;
  const size_t T = cfg->max_tokens;
  auto bail = [&](moe_status_t st) {
    free_layer(L);
    return st;
  };
#define C_TRY(x)                                \
  do {                                          \
    moe_status_t _s = (x);                      \
    if (_s != MOE_OK) return bail(_s);          \
  } while (0)
#define C_CUDA(call)                                                                           \
  do {                                                                                         \
    cudaError_t _e = (call);                                                                   \
    if (_e != cudaSuccess) {                                                                   \
      return bail(fail(MOE_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(_e)));     \
    }                                                                                          \
  } while (0)

  // pinned store in device layout
  const size_t bytes = L->L.bytes;
  if (cudaHostAlloc((void **)&L->store, bytes * E, cudaHostAllocDefault) != cudaSuccess) {
    (void)cudaGetLastError();
    L->store = nullptr;
    return bail(fail(MOE_ERR_OOM, "pinned host store allocation failed"));
  }
  {
    const int nth = std::max(1, std::min<int>(8, (int)std::thread::hardware_concurrency()));
    std::vector<std::thread> th;
    for (int t = 0; t < nth; ++t)
      th.emplace_back([&, t] {
        for (int e = t; e < E; e += nth) pack_expert(cfg, L->L, w, e, L->store + (size_t)e * bytes);
      });
    for (auto &x : th) x.join();
  }
  if (cudaHostAlloc((void **)&L->h_counts, sizeof(int) * E, cudaHostAllocDefault) != cudaSuccess ||
      cudaHostAlloc((void **)&L->h_loc, sizeof(int) * E, cudaHostAllocDefault) != cudaSuccess ||
      cudaHostAlloc((void **)&L->h_err, sizeof(int), cudaHostAllocMapped) != cudaSuccess) {
    (void)cudaGetLastError();
    return bail(fail(MOE_ERR_OOM, "pinned host allocation failed"));
  }

  // device memory
  // router rows: the E experts, the sinks, then the shared-expert gate row
  const int NT = n_targets(cfg), NR = n_logit_rows(cfg);
  C_TRY(dalloc(L, &L->router_w, (size_t)NR * H * 4));
  if (w->router_bias) C_TRY(dalloc(L, &L->router_b, (size_t)NR * 4));
  if (Is) for (int m = 0; m < 3; ++m) C_TRY(dalloc(L, &L->shared_w[m], (size_t)Is * H * 2));
  if (cfg->n_slots) C_TRY(dalloc(L, &L->slots, bytes * cfg->n_slots));
  if (L->n_staging) C_TRY(dalloc(L, &L->staging, bytes * L->n_staging));
  C_TRY(dalloc(L, &L->loc_resident, sizeof(int) * E));
  C_TRY(dalloc(L, &L->loc_pass, sizeof(int) * E));
  C_TRY(dalloc(L, &L->logits, T * NR * 4));
  C_TRY(dalloc(L, &L->ids, z.P * 4));
  C_TRY(dalloc(L, &L->gates, z.P * 4));
  C_TRY(dalloc(L, &L->perm, z.P * 4));
  C_TRY(dalloc(L, &L->inv, z.P * 4));
  C_TRY(dalloc(L, &L->counts, (size_t)NT * 4));
  C_TRY(dalloc(L, &L->offsets, (size_t)(NT + 1) * 4));
  C_TRY(dalloc(L, &L->tiles, z.max_tiles * sizeof(TileInfo)));
  C_TRY(dalloc(L, &L->n_tiles, 4));
  C_TRY(dalloc(L, &L->active, 4));
  const size_t prow_cap = cfg->numerics == MOE_NUMERICS_A4 ? std::max(z.max_prows, z.a4_rows) : z.max_prows;
  C_TRY(dalloc(L, &L->prow_token, prow_cap * 4));
  C_TRY(dalloc(L, &L->prow_pair, prow_cap * 4));
  C_TRY(dalloc(L, &L->xf16, T * H * 2));
  C_TRY(dalloc(L, &L->xs, T * (H / kChunk) * 4));
  C_TRY(dalloc(L, &L->hbuf, z.max_prows * I * 2));
  C_TRY(dalloc(L, &L->hscale, z.max_prows * (I / kChunk) * 4));
  C_TRY(dalloc(L, &L->oprime, z.P * H * 4));
  if (Is) {
    C_TRY(dalloc(L, &L->sh_h, T * Is * 2));
    C_TRY(dalloc(L, &L->sh_s, T * H * 4));
  }
  C_TRY(dalloc(L, &L->router_counter, ((T + 3) / 4) * 4));
  C_TRY(dalloc(L, &L->tiles_done, 4));
  C_TRY(dalloc(L, &L->comb_cnt, T * (H / 128) * 4));
  if (T >= (size_t)kDenseTcMinTokens) C_TRY(dalloc(L, &L->router_parts, kRouterPartFloats * 4));
  if (Is) {
    C_TRY(make_bf16_map(&L->sh_map[0], L->shared_w[0], H, Is));
    C_TRY(make_bf16_map(&L->sh_map[1], L->shared_w[1], H, Is));
    C_TRY(make_bf16_map(&L->sh_map[2], L->shared_w[2], Is, H));
    C_TRY(make_bf16_map(&L->sh_hmap, L->sh_h, Is, T));
  }
  C_TRY(dalloc(L, &L->xin, T * H * 2));
  L->a4 = cfg->numerics == MOE_NUMERICS_A4;
  if (L->a4) {
    const size_t R = z.a4_rows, G = L->L.G;
    L->a4_rows = R;
    C_TRY(dalloc(L, &L->xq, R * H / 2));
    C_TRY(dalloc(L, &L->xsf, R * H / G));
    C_TRY(dalloc(L, &L->xG, R * 4));
    C_TRY(dalloc(L, &L->h32, R * I * 4));
    C_TRY(dalloc(L, &L->hq, R * I / 2));
    C_TRY(dalloc(L, &L->hsf, R * I / G));
    C_TRY(dalloc(L, &L->hG, R * 4));
    C_TRY(dalloc(L, &L->n_prows, 4));
    C_TRY(dalloc(L, &L->a4_work, kWorkCtrs * sizeof(int)));
    C_CUDA(cudaMemsetAsync(L->a4_work, 0, kWorkCtrs * sizeof(int), s));
    C_TRY(make_a4_act_map(&L->a4maps.act[0], L->xq, H / 2, R));
    C_TRY(make_a4_act_map(&L->a4maps.act[1], L->hq, I / 2, R));
  }
  L->tc = uses_tc(cfg);
  {
    int nsm = 0;
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, cfg->device) == cudaSuccess && nsm > 0)
      L->n_sms = nsm;
  }
  if (L->tc) {
    const size_t R = z.tc_tiles * kTcSlotRows;
    L->tc_rows = R;
    C_TRY(dalloc(L, &L->txq, R * H));
    C_TRY(dalloc(L, &L->txsf, R * H / 32));
    C_TRY(dalloc(L, &L->thq, R * I));
    C_TRY(dalloc(L, &L->thsf, R * I / 32));
    C_CUDA(cudaMemsetAsync(L->txq, 0, R * H, s));
    C_CUDA(cudaMemsetAsync(L->txsf, 127, R * H / 32, s));
    C_CUDA(cudaMemsetAsync(L->thq, 0, R * I, s));
    C_CUDA(cudaMemsetAsync(L->thsf, 127, R * I / 32, s));
    C_TRY(dalloc(L, &L->tc_work, kWorkCtrs * sizeof(int)));
    C_CUDA(cudaMemsetAsync(L->tc_work, 0, kWorkCtrs * sizeof(int), s));
    C_TRY(dalloc(L, &L->tile_done, z.tc_tiles * sizeof(int)));
    C_CUDA(cudaMemsetAsync(L->tile_done, 0, z.tc_tiles * sizeof(int), s));
    C_TRY(make_piece_map(&L->tc_act[0], L->txq, H, R));
    C_TRY(make_piece_map(&L->tc_act[1], L->thq, I, R));
  }
  L->nv = uses_dq(cfg);
  if (L->nv) {
    C_TRY(dalloc(L, &L->dq_work, kWorkCtrs * sizeof(int)));
    C_CUDA(cudaMemsetAsync(L->dq_work, 0, kWorkCtrs * sizeof(int), s));
    // x rows gathered into the padded expert order (and their f16 scales)
    C_TRY(dalloc(L, &L->xg, z.max_prows * H * 2));
    C_TRY(dalloc(L, &L->xgs, z.max_prows * 4));
    if (!L->n_prows) C_TRY(dalloc(L, &L->n_prows, 4));
  }
  C_TRY(dalloc(L, &L->yout, T * H * 4));

  C_CUDA(cudaMemsetAsync(L->router_counter, 0, ((T + 3) / 4) * 4, s));
  C_CUDA(cudaMemsetAsync(L->tiles_done, 0, 4, s));
  C_CUDA(cudaMemsetAsync(L->comb_cnt, 0, T * (H / 128) * 4, s));
  C_CUDA(cudaMemsetAsync(L->loc_resident, 0xFF, sizeof(int) * E, s));   // -1: absent
  C_CUDA(cudaMemsetAsync(L->loc_pass, 0xFF, sizeof(int) * E, s));
  *L->h_err = 0;
  {
    ErrWord ew{};
    C_CUDA(cudaHostGetDevicePointer((void **)&ew.host, L->h_err, 0));
    C_TRY(dalloc(L, &L->d_err, sizeof(ErrWord)));
    C_CUDA(cudaMemcpyAsync(L->d_err, &ew, sizeof ew, cudaMemcpyHostToDevice, s));
    C_CUDA(cudaStreamSynchronize(s));                  // ew lives on this stack frame
  }
  for (int m = 0; m < 3; ++m) {
    const int box_rows = m < 2 ? 128 : 256;
    if (cfg->n_slots) C_TRY(make_code_map(&L->maps.slot[m], L->slots, cfg->n_slots, L->L, m, box_rows));
    if (L->n_staging) C_TRY(make_code_map(&L->maps.stage[m], L->staging, L->n_staging, L->L, m, box_rows));
    // A4: gate and up are one interleaved matrix of 2I rows (map 0); down is map 2
    if (L->a4 && m != 1 && cfg->n_slots)
      C_TRY(make_a4_weight_map(&L->a4maps.w[0][m], L->slots, cfg->n_slots, L->L, m));
    if (L->a4 && m != 1 && L->n_staging)
      C_TRY(make_a4_weight_map(&L->a4maps.w[1][m], L->staging, L->n_staging, L->L, m));
    // dequantising kernels: one 64-element K slab per box (32 bytes of nibbles, or 64 FP8 bytes)
    const int dq_box = cfg->fmt == MOE_FMT_FP8B128 ? 64 : 32;
    if (L->nv && cfg->n_slots)
      C_TRY(make_code_map(&L->dqmaps.slot[m], L->slots, cfg->n_slots, L->L, m, box_rows, dq_box));
    if (L->nv && L->n_staging)
      C_TRY(make_code_map(&L->dqmaps.stage[m], L->staging, L->n_staging, L->L, m, box_rows, dq_box));
  }
  if (L->tc) {
    for (int g = 0; g < 2; ++g) {
      if (cfg->n_slots) C_TRY(make_tc_weight_map(&L->tcmaps.w[0][g], L->slots, cfg->n_slots, L->L, g == 0));
      if (L->n_staging) C_TRY(make_tc_weight_map(&L->tcmaps.w[1][g], L->staging, L->n_staging, L->L, g == 0));
    }
  }
  C_CUDA(cudaMemcpyAsync(L->router_w, w->router_w, (size_t)NT * H * 4, cudaMemcpyHostToDevice, s));
  if (cfg->shared_gate)
    C_CUDA(cudaMemcpyAsync(L->router_w + (size_t)NT * H, w->shared_gate_w, (size_t)H * 4, cudaMemcpyHostToDevice, s));
  if (w->router_bias) {
    C_CUDA(cudaMemcpyAsync(L->router_b, w->router_bias, (size_t)NT * 4, cudaMemcpyHostToDevice, s));
    if (cfg->shared_gate) C_CUDA(cudaMemsetAsync(L->router_b + NT, 0, sizeof(float), s));   // the gate row has no bias
  }
  if (Is)
    for (int m = 0; m < 3; ++m)
      C_CUDA(cudaMemcpyAsync(L->shared_w[m], w->shared_w[m], (size_t)Is * H * 2, cudaMemcpyHostToDevice, s));
  C_CUDA(cudaStreamSynchronize(s));

  C_CUDA(cudaStreamCreateWithFlags(&L->side, cudaStreamNonBlocking));
  if (Is) {
    C_CUDA(cudaStreamCreateWithFlags(&L->sh_stream, cudaStreamNonBlocking));
    C_CUDA(cudaEventCreateWithFlags(&L->ev_sh_fork, cudaEventDisableTiming));
    C_CUDA(cudaEventCreateWithFlags(&L->ev_sh_join, cudaEventDisableTiming));
  }
  for (int i = 0; i < 2; ++i) {
    C_CUDA(cudaEventCreateWithFlags(&L->ev_copied[i], cudaEventDisableTiming));
    C_CUDA(cudaEventCreateWithFlags(&L->ev_done[i], cudaEventDisableTiming));
  }
  C_CUDA(cudaEventCreateWithFlags(&L->ev_counts, cudaEventDisableTiming));
  C_CUDA(cudaEventCreateWithFlags(&L->ev_fwd_done, cudaEventDisableTiming));
  C_CUDA(cudaEventCreateWithFlags(&L->ev_prefetch, cudaEventDisableTiming));
  L->slot_of.assign(E, -1);
  L->expert_of_slot.assign(cfg->n_slots, -1);
  L->last_use.assign(E, 0);
  L->st.expert_bytes = bytes;
  L->st.pinned_bytes = bytes * E;
  size_t dev_total = (size_t)NR * H * 4 + (size_t)3 * Is * H * 2 + bytes * (cfg->n_slots + L->n_staging) +
                     scratch_bytes(cfg) + a4_scratch_bytes(cfg) + tc_scratch_bytes(cfg);
  L->st.device_bytes = dev_total;
  *out = L;
  return MOE_OK;
#undef C_TRY
#undef C_CUDA
}

moe_status_t moe_set_slot_table(moe_layer_t L, const int32_t *table, void *stream) {
  if (!L || !table) return fail(MOE_ERR_INVALID_ARG, "layer or table is NULL");
  const int E = L->cfg.n_experts, S = L->cfg.n_slots;
  std::vector<int> used(S > 0 ? S : 1, -1);
  int n = 0;
  for (int e = 0; e < E; ++e) {
    const int s = table[e];
    if (s == -1) continue;
    if (s < 0 || s >= S) {
      char buf[96];
      snprintf(buf, sizeof buf, "slot %d of expert %d is out of range [0, %d)", s, e, S);
      return fail(MOE_ERR_SLOT_TABLE, buf);
    }
    if (used[s] >= 0) {
      char buf[96];
      snprintf(buf, sizeof buf, "slot %d given to experts %d and %d", s, used[s], e);
      return fail(MOE_ERR_SLOT_TABLE, buf);
    }
    used[s] = e;
    ++n;
  }
  if (n > S) return fail(MOE_ERR_SLOT_TABLE, "more resident experts than slots");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  cudaStream_t st = (cudaStream_t)stream;
  CUDA_TRY(cudaStreamSynchronize(st));
  CUDA_TRY(cudaStreamSynchronize(L->side));
  const size_t bytes = L->L.bytes;
  for (int e = 0; e < E; ++e) {
    const int s = table[e];
    if (s >= 0 && L->slot_of[e] != s)
      CUDA_TRY(cudaMemcpyAsync(L->slots + (size_t)s * bytes, L->store + (size_t)e * bytes, bytes,
                               cudaMemcpyHostToDevice, st));
    L->h_loc[e] = s >= 0 ? s : kLocAbsent;
  }
  CUDA_TRY(cudaMemcpyAsync(L->loc_resident, L->h_loc, sizeof(int) * E, cudaMemcpyHostToDevice, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  for (int e = 0; e < E; ++e) L->slot_of[e] = table[e];
  std::fill(L->expert_of_slot.begin(), L->expert_of_slot.end(), -1);
  for (int e = 0; e < E; ++e)
    if (table[e] >= 0) L->expert_of_slot[table[e]] = e;
  L->n_resident = n;
  L->table_version += 1;
  return MOE_OK;
}

// Index ranges of the forward being enqueued, for the device bounds checks of
// the checked build.
static DevBounds dev_bounds(const moe_layer *L) {
  DevBounds b;
  b.n_experts = L->cfg.n_experts;
  b.n_targets = n_targets(&L->cfg);
  b.n_slots = L->cfg.n_slots;
  b.n_staging = L->n_staging;
  b.n_tokens = L->cur_T;
  b.n_pairs = L->cur_T * L->cfg.top_k;
  b.err = L->d_err;
  return b;
}

// K split (cluster size) of the register-decode passes, a power of two up to 8
// that divides the chunk count.  Gate/up doubles it while its items number
// fewer than two per SM (it may end with up to twice that); the down pass only
// while they still fit one round of two CTAs per SM.  Measured on the
// Qwen3.8-Flash-Next-like layer: the down rule took the T = 1 step from 74.1
// to 68.1 us and T = 3 from 100.5 to 97.9 us; the same cap on gate/up saved
// 8 us at T = 1 but cost 9.5 us at T = 2 (split 2 -> 1), so gate/up keeps
// the looser rule.
static int pick_split(int est_ctas, int nck) {
  int cs = 1;
  while (cs < 8 && nck % (cs * 2) == 0 && est_ctas * cs < 2 * 148) cs *= 2;
  return cs;
}
static int pick_split_fit(int est_ctas, int nck) {
  int cs = 1;
  while (cs < 8 && nck % (cs * 2) == 0 && est_ctas * cs * 2 <= 2 * 148) cs *= 2;
  return cs;
}

// The stream waits for the shared expert forked onto its own stream (once per
// forward, before the first kernel that reads the shared expert's output).
static moe_status_t join_shared(moe_layer *L, cudaStream_t s) {
  if (!L->sh_join_pending) return MOE_OK;
  L->sh_join_pending = false;
  CUDA_TRY(cudaStreamWaitEvent(s, L->ev_sh_join, 0));
  return MOE_OK;
}

static moe_status_t run_experts(moe_layer *L, const int *locs, int nt, int grid_tiles, int cs_gu, int cs_dn,
                                float *y, cudaStream_t s) {
  const moe_config_t &c = L->cfg;
  TmaExpertArgs a{};
  a.db = dev_bounds(L);
  a.maps = L->maps;
  a.loc = locs;
  a.slots = L->slots;
  a.staging = L->staging;
  a.blob_bytes = L->L.bytes;
  a.L = L->L;
  a.tile_tokens = 8 * nt;
  a.tiles = L->tiles;
  a.n_tiles = L->n_tiles;
  a.prow_token = L->prow_token;
  a.prow_pair = L->prow_pair;
  a.gates = L->gates;
  a.err = L->d_err;
  a.y = y;
  a.shared = c.shared_inter ? L->sh_s : nullptr;
  a.comb_cnt = L->comb_cnt;
  a.top_k = c.top_k;
  // gate/up + SwiGLU
  a.K = c.hidden;
  a.rows = c.inter;
  a.n_rowblocks = c.inter / 128;
  a.k_split = cs_gu;
  a.act = L->xf16;
  a.act_scale = L->xs;
  a.h_out = L->hbuf;
  a.h_scale = L->hscale;
  StageTimer t3(L, 3, s);
  launch_expert_tma(L->wf, MODE_GATEUP, nt, a, grid_tiles, s);
  CUDA_TRY(cudaGetLastError());
  t3.launched(1);
  t3.end();
  // down + gate scale -> O'
  a.K = c.inter;
  a.rows = c.hidden;
  a.n_rowblocks = c.hidden / 256;
  a.k_split = cs_dn;
  a.act = L->hbuf;
  a.act_scale = L->hscale;
  a.o_out = L->oprime;
  // the down pass adds the shared expert's output when it runs the combine
  if (y) ST_TRY(join_shared(L, s));
  StageTimer t4(L, 4, s);
  launch_expert_tma(L->wf, MODE_DOWN, nt, a, grid_tiles, s);
  CUDA_TRY(cudaGetLastError());
  t4.launched(1);
  t4.end();
  return MOE_OK;
}

// Tensor-core EXACT pass over the experts present in `locs`: gate/up + SwiGLU
// -> h pieces, down + gate -> O' and the ordered combine into y.
static moe_status_t run_experts_tc(moe_layer *L, const int *locs, int nbox, int grid_tiles, cudaStream_t s) {
  const moe_config_t &c = L->cfg;
  TcArgs a{};
  a.db = dev_bounds(L);
  a.maps = L->tcmaps;
  a.loc = locs;
  a.slots = L->slots;
  a.staging = L->staging;
  a.blob_bytes = L->L.bytes;
  a.L = L->L;
  a.tiles = L->tiles;
  a.n_tiles = L->n_tiles;
  a.prow_pair = L->prow_pair;
  a.gates = L->gates;
  a.err = L->d_err;
  a.hq = L->thq;
  a.hsf = L->thsf;
  a.o_out = L->oprime;
  a.act = L->txq;
  a.maps.act = L->tc_act[0];
  a.K = c.hidden;
  a.rows = c.inter;
  a.n_rowblocks = c.inter / 128;
  a.bsf = L->txsf;
  a.work_ctr = L->tc_work;
  a.grid = std::min(grid_tiles * a.n_rowblocks, L->n_sms);
  a.early = locs == L->loc_resident ? 1 : 0;
  // decode tiles, all resident: the down pass takes each tile's h as soon as
  // the gate/up items of that tile are done (counters zeroed by the routing step)
  a.tile_done = (a.early && nbox <= 16) ? L->tile_done : nullptr;
  a.tile_target = c.inter / 128;
  StageTimer t3(L, 3, s);
  launch_expert_tc(MODE_GATEUP, nbox, a, grid_tiles, s);
  CUDA_TRY(cudaGetLastError());
  t3.launched(1);
  t3.end();
  a.act = L->thq;
  a.maps.act = L->tc_act[1];
  a.K = c.inter;
  a.rows = c.hidden;
  a.n_rowblocks = c.hidden / 256;
  a.bsf = L->thsf;
  a.work_ctr = L->tc_work + 1;
  a.grid = std::min(grid_tiles * a.n_rowblocks, L->n_sms);
  // the down pass starts its weight stream before the gate/up pass ends only
  // with decode-sized tiles (there the gate/up CTAs end at different times);
  // with prefill tiles this measured several times slower
  a.early = (a.early && nbox <= 16) ? 1 : 0;
  StageTimer t4(L, 4, s);
  launch_expert_tc(MODE_DOWN, nbox, a, grid_tiles, s);
  CUDA_TRY(cudaGetLastError());
  t4.launched(1);
  t4.end();
  return MOE_OK;
}

// NVFP4 EXACT pass on the tensor core over the experts present in `locs`
// (tiles of nb tokens): gate/up + SwiGLU -> h (bf16, padded-row order), then
// down + gate -> O'; the ordered combine follows after the last pass.
static moe_status_t run_experts_dq(moe_layer *L, const int *locs, const void *x, int nb, int grid_tiles,
                                   cudaStream_t s) {
  const moe_config_t &c = L->cfg;
  DqArgs a{};
  a.db = dev_bounds(L);
  a.maps = L->dqmaps;
  a.loc = locs;
  a.slots = L->slots;
  a.staging = L->staging;
  a.blob_bytes = L->L.bytes;
  a.L = L->L;
  a.tiles = L->tiles;
  a.n_tiles = L->n_tiles;
  a.prow_token = L->prow_token;
  a.prow_pair = L->prow_pair;
  a.gates = L->gates;
  a.err = L->d_err;
  a.K = c.hidden;
  a.rows = c.inter;
  a.n_rowblocks = c.inter / 128;
  // NVFP4: x as f16 rows with a power-of-two scale per token (written into
  // the f16 activation buffer by the conversion before the first pass)
  const bool f16x = c.fmt == MOE_FMT_NVFP4;
  (void)x;
  a.act = L->xg;                                   // x rows gathered into the padded expert order
  a.act_scale = f16x ? L->xgs : nullptr;
  ST_TRY(make_bf16_map(&a.maps.act, L->xg, c.hidden, L->max_prows, 64));
  a.h_out = L->hbuf;
  a.work_ctr = L->dq_work;
  a.wfmt = c.fmt == MOE_FMT_INT4G128 ? DQ_I4 : (c.fmt == MOE_FMT_FP8B128 ? DQ_F8 : DQ_NV);
  a.grid = std::min(grid_tiles * a.n_rowblocks, L->n_sms);
  StageTimer t3(L, 3, s);
  launch_expert_dq(MODE_GATEUP, nb, a, s);
  CUDA_TRY(cudaGetLastError());
  t3.launched(1);
  t3.end();
  a.K = c.inter;
  a.rows = c.hidden;
  a.n_rowblocks = c.hidden / 256;
  a.act = L->hbuf;
  a.act_scale = nullptr;
  ST_TRY(make_bf16_map(&a.maps.act, L->hbuf, c.inter, L->max_prows, 64));
  a.o_out = L->oprime;
  a.work_ctr = L->dq_work + 1;
  a.grid = std::min(grid_tiles * a.n_rowblocks, L->n_sms);
  StageTimer t4(L, 4, s);
  launch_expert_dq(MODE_DOWN, nb, a, s);
  CUDA_TRY(cudaGetLastError());
  t4.launched(1);
  t4.end();
  return MOE_OK;
}

// A4 pass over the experts present in `locs`: tcgen05 gate/up + SwiGLU -> h fp32,
// quantise h rows of these experts, tcgen05 down + gate -> O'.
static moe_status_t run_experts_a4(moe_layer *L, const int *locs, int grid_tiles, cudaStream_t s) {
  const moe_config_t &c = L->cfg;
  A4GemmArgs g{};
  g.db = dev_bounds(L);
  g.maps = L->a4maps;
  g.loc = locs;
  g.slots = L->slots;
  g.staging = L->staging;
  g.blob_bytes = L->L.bytes;
  g.L = L->L;
  g.tiles = L->tiles;
  g.n_tiles = L->n_tiles;
  g.prow_pair = L->prow_pair;
  g.gates = L->gates;
  g.err = L->d_err;
  g.act_map = 0;
  g.K = c.hidden;
  g.rows = c.inter;
  g.n_rowblocks = c.inter / 64;                 // 64 h columns (gate + up rows) per item
  g.work_ctr = L->a4_work;
  g.grid = std::min(grid_tiles * g.n_rowblocks, L->n_sms);
  g.bsf = L->xsf;
  g.bG = L->xG;
  g.h_out = L->h32;
  // MXFP4: the gate/up epilogue quantises h itself (its block scale is local
  // to 32 columns of one token); NVFP4's per-row tensor scale needs the whole
  // row first, so there h goes through fp32 and the quantiser
  const bool fuse_hq = c.fmt == MOE_FMT_MXFP4;
  g.hq_out = fuse_hq ? L->hq : nullptr;
  g.hsf_out = fuse_hq ? L->hsf : nullptr;
  StageTimer t3(L, 3, s);
  launch_gemm_a4(L->wf, MODE_GATEUP, g, s);
  CUDA_TRY(cudaGetLastError());
  t3.launched(1);
  t3.end();
  if (!fuse_hq) {
    StageTimer t8(L, 8, s);
    QuantArgs q{};
    q.db = dev_bounds(L);
    q.max_rows = (int)L->a4_rows;
    q.n_rows = L->n_prows;
    q.K = c.inter;
    q.fmt = c.fmt;
    q.src_f32 = L->h32;
    q.row_pair = L->prow_pair;
    q.loc = locs;
    q.ids = L->ids;
    q.codes = L->hq;
    q.sf = L->hsf;
    q.G = L->hG;
    launch_quant(q, s);
    CUDA_TRY(cudaGetLastError());
    t8.launched(1);
    t8.end();
  }
  g.hq_out = nullptr;
  g.hsf_out = nullptr;
  g.act_map = 1;
  g.K = c.inter;
  g.rows = c.hidden;
  g.n_rowblocks = c.hidden / 128;
  g.work_ctr = L->a4_work + 1;
  g.grid = std::min(grid_tiles * g.n_rowblocks, L->n_sms);
  g.bsf = L->hsf;
  g.bG = L->hG;
  g.o_out = L->oprime;
  StageTimer t4(L, 4, s);
  launch_gemm_a4(L->wf, MODE_DOWN, g, s);
  CUDA_TRY(cudaGetLastError());
  t4.launched(1);
  t4.end();
  return MOE_OK;
}

moe_status_t moe_forward(moe_layer_t L, const void *x, int32_t T, void *y, void *stream,
                         const moe_routing_t *dbg) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  const moe_config_t &c = L->cfg;
  if (T < 0 || T > c.max_tokens) return fail(MOE_ERR_INVALID_ARG, "T out of range [0, max_tokens]");
  if (T == 0) return MOE_OK;
  if (!x || !y) return fail(MOE_ERR_INVALID_ARG, "x or y is NULL");
  if (*(volatile int *)L->h_err != 0) return report_device_error(L, stream);
  if (L->inject == 3) {
    // test hook: the device error word is set before this forward's kernels
    // run, so that every bounded wait of theirs that has to wait gives up
    // at once (the path a wait takes when its time limit passes)
    L->inject = 0;
    *(volatile int *)L->h_err = 99;
    CUDA_TRY(cudaMemsetAsync(L->d_err, 0x63, sizeof(int), (cudaStream_t)stream));
  }
  CUDA_TRY(cudaSetDevice(c.device));
  cudaStream_t s = (cudaStream_t)stream;
  const int E = c.n_experts, k = c.top_k, H = c.hidden, I = c.inter, Is = c.shared_inter;
  const int P = T * k;
  L->cur_T = T;
  const int act_est = std::min(E, P);
  const int avg = (P + act_est - 1) / act_est;
  const int nt = avg <= 8 ? 1 : (avg <= 16 ? 2 : 4);
  const bool a4 = L->a4;
  const bool tc = L->tc;
  // tensor-core EXACT: 8-token tiles (16 piece rows, 6 stages in flight) while
  // the batch is decode-sized, else 56-token tiles (112 piece rows, two
  // accumulator buffers so that the epilogue overlaps the next item's MMAs)
  const int nbox = (tc && P <= 12 * act_est) ? 16 : 112;
  // NVFP4 EXACT: prefill-sized batches (x 16-byte aligned for the 16-byte
  // activation copies) on the tensor core with tiles of 64 or 128 tokens;
  // decode-sized batches on the register-decode kernels
  const bool x16 = (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  if (dq_only(&c) && !x16) return fail(MOE_ERR_INVALID_ARG, "x must be 16-byte aligned for INT4 / FP8 experts");
  const bool dq = L->nv && (dq_only(&c) || P > 12 * act_est) && x16;
  // 128-token tiles once experts average more than 16 tokens: a weight slab
  // decoded into TMEM then serves twice the tokens, and the pass is bound by
  // the bytes each SM pulls through L2 per MMA (measured on the
  // Qwen3.8-Flash-Next-like layer: at 40 tokens per expert, gate/up 0.98 ms
  // with 64-token tiles, 0.74 ms with 128); 64-token tiles (two accumulator
  // buffers) for decode-sized batches, where an expert's rows fit one tile
  const int nb_dq = avg > 16 ? 128 : 64;
  const int ts = a4 ? 128 : (tc ? nbox / 2 : (dq ? nb_dq : 8 * nt));
  const int grid_tiles = P / ts + act_est + 1;
  // routing targets (experts, then sinks) and logit rows (+ the shared-expert gate)
  const int NT = n_targets(&c), NR = n_logit_rows(&c);
  // the register-decode kernels fuse the ordered combine into their down pass
  // for fp32 outputs of layers without sinks or a shared-expert gate; every
  // other case runs the combine kernel after the last pass
  const bool sep_combine = a4 || tc || dq || c.n_sinks > 0 || c.shared_gate || c.out_dtype == MOE_OUT_BF16;
  float *y_fused = sep_combine ? nullptr : static_cast<float *>(y);

  StageTimer t7(L, 7, s);
  // decode-sized batches: the shared expert reads only x, so it runs on its
  // own stream beside the routing and the routed passes (its split-K clusters
  // and the routed kernels are each too short to keep HBM busy alone)
  const bool sh_fork = Is && T <= 128;
  L->sh_join_pending = false;
  if (sh_fork) CUDA_TRY(cudaEventRecord(L->ev_sh_fork, s));
  // every return from here on, an error return included, leaves `s` ordered
  // after the work this forward queued on the shared expert's stream
  struct SharedJoinGuard {
    moe_layer *L;
    cudaStream_t s;
    ~SharedJoinGuard() {
      if (!L->sh_join_pending) return;
      L->sh_join_pending = false;
      cudaEventRecord(L->ev_sh_join, L->sh_stream);
      cudaStreamWaitEvent(s, L->ev_sh_join, 0);
    }
  } sh_guard{L, s};
  RouterArgs ra{};
  ra.x = reinterpret_cast<const uint16_t *>(x);
  ra.T = T; ra.H = H; ra.E = NR; ra.k = k;
  ra.E_t = NT; ra.scoring = c.scoring; ra.renorm = c.renormalize;
  ra.w = L->router_w; ra.bias = L->router_b;
  ra.logits = L->logits; ra.ids = L->ids; ra.gates = L->gates;
  ra.xf16 = tc ? nullptr : L->xf16; ra.xs = L->xs; ra.counter = L->router_counter;
  PermArgs pa{};
  pa.db = dev_bounds(L);
  pa.ids = L->ids; pa.n_pairs = P; pa.E = NT; pa.n_real = E; pa.k = k; pa.tile_tokens = ts;
  pa.counts = L->counts; pa.offsets = L->offsets; pa.perm = L->perm; pa.inv = L->inv;
  pa.tiles = L->tiles; pa.n_tiles = L->n_tiles; pa.prow_token = L->prow_token;
  pa.prow_pair = L->prow_pair; pa.active = L->active;
  pa.pad = a4 ? 128 : 8;
  pa.n_prows = (a4 || dq) ? L->n_prows : nullptr;
  pa.work_ctr = tc ? L->tc_work : (dq ? L->dq_work : (a4 ? L->a4_work : nullptr));
  pa.tile_done = tc ? L->tile_done : nullptr;
  // decode-sized batches: the router's last CTA also runs the permutation
  const bool fuse_perm = P <= 2048;
  ra.fuse_perm = fuse_perm ? 1 : 0;
  ra.tiles_done = L->tiles_done;
  ra.perm = pa;
  // prefill-sized batches: logits by a tiled GEMM, then top-k and the
  // permutation as their own kernels (the register-decode kernels of NVFP4
  // EXACT layers need the router's f16 copy of x, so they keep the router)
  const bool big_batch = T >= kDenseTcMinTokens && (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
  const bool router_gemm = big_batch && (tc || a4 || dq);
  StageTimer t0(L, 0, s);
  if (router_gemm) {
    const int sp = router_gemm_splits(T, H, NR, kRouterPartFloats);
    launch_router_gemm(ra.x, L->router_w, L->router_b, T, H, NR, L->logits, L->router_parts, sp, s);
    CUDA_TRY(cudaGetLastError());
    launch_topk(L->logits, L->router_parts, sp, L->router_b, T, NR, NT, k, c.scoring, c.renormalize, L->ids,
                L->gates, s);
    t0.launched(1);
  } else {
    launch_router(ra, s);
  }
  CUDA_TRY(cudaGetLastError());
  t0.launched(1);
  t0.end();
  if (!fuse_perm || router_gemm) {
    StageTimer t1(L, 1, s);
    launch_permute(pa, s);
    CUDA_TRY(cudaGetLastError());
    t1.launched(1);
    t1.end();
  }

  if (dbg) {
    // logits of the NT routing targets (the rows' stride is NR)
    if (dbg->logits)
      CUDA_TRY(cudaMemcpy2DAsync(dbg->logits, (size_t)NT * 4, L->logits, (size_t)NR * 4, (size_t)NT * 4, T,
                                 cudaMemcpyDeviceToDevice, s));
    if (dbg->ids) CUDA_TRY(cudaMemcpyAsync(dbg->ids, L->ids, (size_t)P * 4, cudaMemcpyDeviceToDevice, s));
    if (dbg->gates) CUDA_TRY(cudaMemcpyAsync(dbg->gates, L->gates, (size_t)P * 4, cudaMemcpyDeviceToDevice, s));
    if (dbg->counts) CUDA_TRY(cudaMemcpyAsync(dbg->counts, L->counts, (size_t)NT * 4, cudaMemcpyDeviceToDevice, s));
    if (dbg->offsets)
      CUDA_TRY(cudaMemcpyAsync(dbg->offsets, L->offsets, (size_t)(NT + 1) * 4, cudaMemcpyDeviceToDevice, s));
    if (dbg->perm) CUDA_TRY(cudaMemcpyAsync(dbg->perm, L->perm, (size_t)P * 4, cudaMemcpyDeviceToDevice, s));
    if (dbg->inv) CUDA_TRY(cudaMemcpyAsync(dbg->inv, L->inv, (size_t)P * 4, cudaMemcpyDeviceToDevice, s));
  }

  const bool resident = L->n_resident == E;
  // slots filled by moe_prefetch: the expert passes wait for those copies
  if (L->prefetch_pending) {
    CUDA_TRY(cudaStreamWaitEvent(s, L->ev_prefetch, 0));
    L->prefetch_pending = false;
  }
  if (!resident) {
    CUDA_TRY(cudaMemcpyAsync(L->h_counts, L->counts, (size_t)E * 4, cudaMemcpyDeviceToHost, s));
    CUDA_TRY(cudaEventRecord(L->ev_counts, s));
  }

  // always-resident shared expert (runs while the host builds the miss list),
  // bf16 on the tensor core: decode-sized batches (T <= 128) split K over a
  // thread-block cluster per row block, larger ones run persistent tiles of
  // 128 tokens.  Its operands are read by TMA, which needs x 16-byte aligned:
  // an unaligned x is first copied to the layer's own buffer.
  if (Is) {
    const cudaStream_t ss = sh_fork ? L->sh_stream : s;
    if (sh_fork) {
      CUDA_TRY(cudaStreamWaitEvent(ss, L->ev_sh_fork, 0));
      L->sh_join_pending = true;
    }
    StageTimer t2(L, 2, ss);
    const void *xs = x;
    if (!x16) {
      CUDA_TRY(cudaMemcpyAsync(L->xin, x, (size_t)T * H * 2, cudaMemcpyDeviceToDevice, ss));
      xs = L->xin;
    }
    DenseTcArgs d{};
    d.wmap[0] = L->sh_map[0];
    d.wmap[1] = L->sh_map[1];
    d.T = T; d.K = H; d.rows = Is; d.n_rowblocks = Is / 128;
    d.h_out = L->sh_h;
    d.s_out = L->sh_s;
    d.err = L->d_err;
    if (T <= 128) {
      const int np = dense_splitk_rows(T);
      ST_TRY(make_bf16_map(&d.xmap, xs, H, T, np));
      launch_dense_splitk(MODE_GATEUP, d, ss);
      CUDA_TRY(cudaGetLastError());
      d.wmap[0] = L->sh_map[2];
      ST_TRY(make_bf16_map(&d.xmap, L->sh_h, Is, T, np));
      d.K = Is; d.rows = H; d.n_rowblocks = H / 256;
      launch_dense_splitk(MODE_DOWN, d, ss);
      CUDA_TRY(cudaGetLastError());
    } else {
      ST_TRY(make_bf16_map(&d.xmap, xs, H, T));
      d.grid = std::min(((T + 127) / 128) * d.n_rowblocks, L->n_sms);
      launch_dense_tc(MODE_GATEUP, d, s);
      CUDA_TRY(cudaGetLastError());
      d.wmap[0] = L->sh_map[2];
      d.xmap = L->sh_hmap;
      d.K = Is; d.rows = H; d.n_rowblocks = H / 256;
      d.grid = std::min(((T + 127) / 128) * d.n_rowblocks, L->n_sms);
      launch_dense_tc(MODE_DOWN, d, s);
      CUDA_TRY(cudaGetLastError());
    }
    t2.launched(2);
    t2.end();
    if (sh_fork) CUDA_TRY(cudaEventRecord(L->ev_sh_join, ss));
  }

  if (a4) {
    QuantArgs q{};
    q.db = dev_bounds(L);
    q.max_rows = (int)L->a4_rows;
    q.n_rows = L->n_prows;
    q.K = H;
    q.fmt = c.fmt;
    q.src_bf16 = reinterpret_cast<const uint16_t *>(x);
    q.row_token = L->prow_token;
    q.codes = L->xq;
    q.sf = L->xsf;
    q.G = L->xG;
    StageTimer tq(L, 8, s);
    launch_quant(q, s);
    CUDA_TRY(cudaGetLastError());
    tq.launched(1);
    tq.end();
  }
  if (tc) {
    TcQuantArgs q{};
    q.db = dev_bounds(L);
    q.x = reinterpret_cast<const uint16_t *>(x);
    q.H = H;
    q.tiles = L->tiles;
    q.n_tiles = L->n_tiles;
    q.max_tiles = grid_tiles;
    q.tile_tokens = ts;
    q.prow_token = L->prow_token;
    q.xq = L->txq;
    q.xsf = L->txsf;
    StageTimer tq(L, 8, s);
    launch_tc_quant_x(q, s);
    CUDA_TRY(cudaGetLastError());
    tq.launched(1);
    tq.end();
  }
  if (dq) {
    // the dequantising pass reads x in the padded expert order, one box per
    // slab; NVFP4 multiplies gate/up in f16 (rows with a power-of-two scale)
    StageTimer tq(L, 8, s);
    launch_gather_rows(reinterpret_cast<const uint16_t *>(x), H, L->prow_token, L->n_prows, (int)L->max_prows,
                       c.fmt == MOE_FMT_NVFP4 ? 1 : 0, L->xg, L->xgs, dev_bounds(L), s);
    CUDA_TRY(cudaGetLastError());
    tq.launched(1);
    tq.end();
  }
  const int cs_gu = pick_split(act_est * (I / 128), H / 128);
  const int cs_dn = pick_split_fit(act_est * (H / 256), I / 128);
  int waves = 0, misses_n = 0;
  bool admit_table_pending = false;
  if (resident) {
    if (a4) ST_TRY(run_experts_a4(L, L->loc_resident, grid_tiles, s));
    else if (tc) ST_TRY(run_experts_tc(L, L->loc_resident, nbox, grid_tiles, s));
    else if (dq) ST_TRY(run_experts_dq(L, L->loc_resident, x, nb_dq, grid_tiles, s));
    else ST_TRY(run_experts(L, L->loc_resident, nt, grid_tiles, cs_gu, cs_dn, y_fused, s));
  } else {
    CUDA_TRY(cudaEventSynchronize(L->ev_counts));
    std::vector<int> misses;
    int act = 0;
    for (int e = 0; e < E; ++e) {
      if (L->h_counts[e] > 0) {
        ++act;
        if (L->slot_of[e] < 0) misses.push_back(e);
      }
    }
    L->st.last_active = act;
    misses_n = (int)misses.size();
    const int NS = L->n_staging;
    const uint64_t fwd_index = L->st.forwards + 1;
    for (int e = 0; e < E; ++e)
      if (L->h_counts[e] > 0) L->last_use[e] = fwd_index;
    // CACHE / HYBRID: which misses this forward admits, and into which slots
    const std::vector<int> admit_slot = plan_admission(L, misses);
    if (misses.empty()) {
      if (a4) ST_TRY(run_experts_a4(L, L->loc_resident, grid_tiles, s));
      else if (tc) ST_TRY(run_experts_tc(L, L->loc_resident, nbox, grid_tiles, s));
      else if (dq) ST_TRY(run_experts_dq(L, L->loc_resident, x, nb_dq, grid_tiles, s));
      else ST_TRY(run_experts(L, L->loc_resident, nt, grid_tiles, cs_gu, cs_dn, y_fused, s));
    } else {
      const bool one = misses_n <= NS;
      const int wave_sz = one ? NS : NS / 2;
      const int nw = (misses_n + wave_sz - 1) / wave_sz;
      const size_t bytes = L->L.bytes;
      if (L->inject == 1) {   // host-side failure injection: no copy is issued
        L->inject = 0;
        return fail(MOE_ERR_CUDA, "staging copy failed (injected)");
      }
      // the previous forward's kernels must be done with the staging ring
      if (L->staging_used) CUDA_TRY(cudaStreamWaitEvent(L->side, L->ev_fwd_done, 0));
      for (int w = 0; w < nw; ++w) {
        const int half = one ? 0 : (w & 1);
        const int base = one ? 0 : half * (NS / 2);
        if (!one && w >= 2) CUDA_TRY(cudaStreamWaitEvent(L->side, L->ev_done[half], 0));
        LocUpdate u{};
        u.E = E;
        u.work_ctr = tc ? L->tc_work : (dq ? L->dq_work : (a4 ? L->a4_work : nullptr));
        u.keep_resident = (w == 0);
        const int b0 = w * wave_sz, b1 = std::min(misses_n, b0 + wave_sz);
        for (int i = b0; i < b1; ++i) {
          const int e = misses[i];
          uint8_t *dst = L->staging + (size_t)(base + (i - b0)) * bytes;
          CUDA_TRY(cudaMemcpyAsync(dst, L->store + (size_t)e * bytes, bytes, cudaMemcpyHostToDevice, L->side));
          u.expert[u.n] = e;
          u.loc[u.n] = loc_staging(base + (i - b0));
          ++u.n;
        }
        CUDA_TRY(cudaEventRecord(L->ev_copied[half], L->side));
        StageTimer t6(L, 6, s);
        CUDA_TRY(cudaStreamWaitEvent(s, L->ev_copied[half], 0));
        launch_loc_update(u, L->loc_resident, L->loc_pass, s);
        CUDA_TRY(cudaGetLastError());
        t6.launched(1);
        t6.end();
        if (a4) ST_TRY(run_experts_a4(L, L->loc_pass, grid_tiles, s));
        else if (tc) ST_TRY(run_experts_tc(L, L->loc_pass, nbox, grid_tiles, s));
        else if (dq) ST_TRY(run_experts_dq(L, L->loc_pass, x, nb_dq, grid_tiles, s));
        else ST_TRY(run_experts(L, L->loc_pass, nt, grid_tiles, cs_gu, cs_dn, y_fused, s));
        // admissions: the staged copy of an admitted miss goes into its slot
        // while the staging buffer still holds it (a slot whose expert this
        // forward does not use, so no kernel of this forward reads it)
        for (int i = b0; i < b1; ++i)
          if (admit_slot[i] >= 0)
            CUDA_TRY(cudaMemcpyAsync(L->slots + (size_t)admit_slot[i] * bytes,
                                     L->staging + (size_t)(base + (i - b0)) * bytes, bytes,
                                     cudaMemcpyDeviceToDevice, s));
        if (!one) CUDA_TRY(cudaEventRecord(L->ev_done[half], s));
      }
      CUDA_TRY(cudaEventRecord(L->ev_fwd_done, s));
      L->staging_used = true;
      waves = nw;
      L->st.misses += misses_n;
      L->st.bytes_staged += (uint64_t)misses_n * bytes;
      // the admitted experts are resident from the next forward on: the new
      // table reaches the device behind this forward's kernels on the stream
      int admitted = 0;
      for (int i = 0; i < misses_n; ++i) {
        const int v = admit_slot[i];
        if (v < 0) continue;
        const int old = L->expert_of_slot[v];
        if (old >= 0) L->slot_of[old] = -1;
        L->slot_of[misses[i]] = v;
        L->expert_of_slot[v] = misses[i];
        ++admitted;
      }
      if (admitted) {
        L->st.admitted += admitted;
        admit_table_pending = true;
      }
    }
  }

  // the ordered combine: inside the register-decode down pass (last arrival
  // per token) when y_fused is set, else this kernel after the last pass
  if (sep_combine) {
    CombineArgs ca{};
    ca.oprime = L->oprime;
    ca.shared = Is ? L->sh_s : nullptr;
    ca.y = y;
    ca.T = T; ca.H = H; ca.k = k;
    ca.out_bf16 = c.out_dtype == MOE_OUT_BF16 ? 1 : 0;
    ca.ids = c.n_sinks > 0 ? L->ids : nullptr;
    ca.n_real = E;
    ca.sg_logits = c.shared_gate ? L->logits : nullptr;
    ca.ld = NR;
    ca.sg_col = NT;
    ST_TRY(join_shared(L, s));
    StageTimer t5(L, 5, s);
    launch_combine(ca, s);
    CUDA_TRY(cudaGetLastError());
    t5.launched(1);
    t5.end();
  }
  // every path has read the shared output by now; a forward whose passes all
  // fused the combine without one still ends behind the shared stream
  ST_TRY(join_shared(L, s));
  if (admit_table_pending) ST_TRY(push_table(L, s));
  t7.end();
  if (L->prof) L->prof_acc.forwards += 1;

  L->st.forwards += 1;
  L->st.last_misses = misses_n;
  L->st.last_waves = waves;
  L->st.last_path = a4 ? 1 : (tc ? 2 : (dq ? 3 : 0));
  if (resident) L->st.last_active = -1;
  return MOE_OK;
}

moe_status_t moe_forward_host(moe_layer_t L, const uint16_t *x_host, int32_t T, void *y_host,
                              void *stream) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  if (T < 0 || T > L->cfg.max_tokens) return fail(MOE_ERR_INVALID_ARG, "T out of range [0, max_tokens]");
  if (T == 0) return MOE_OK;
  if (!x_host || !y_host) return fail(MOE_ERR_INVALID_ARG, "x or y is NULL");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  cudaStream_t s = (cudaStream_t)stream;
  const size_t H = L->cfg.hidden;
  CUDA_TRY(cudaMemcpyAsync(L->xin, x_host, (size_t)T * H * 2, cudaMemcpyHostToDevice, s));
  ST_TRY(moe_forward(L, L->xin, T, L->yout, stream, nullptr));
  const size_t ybytes = L->cfg.out_dtype == MOE_OUT_BF16 ? 2 : 4;
  CUDA_TRY(cudaMemcpyAsync(y_host, L->yout, (size_t)T * H * ybytes, cudaMemcpyDeviceToHost, s));
  CUDA_TRY(cudaStreamSynchronize(s));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// CUDA-graph capture of one all-resident forward (fixed x, T, y).  The
// resident forward only enqueues kernels (no host synchronisation), so it can
// be captured as it is; a replay runs the same launch chain without the
// per-kernel CPU launch cost.
// ---------------------------------------------------------------------------
struct moe_graph {
  moe_layer *L = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  uint64_t table_version = 0;
  uint64_t launches = 0;             // library kernels per replay
};

moe_status_t moe_graph_capture(moe_layer_t L, const void *x, int32_t T, void *y, void *stream,
                               moe_graph_t *out) {
  if (!L || !out) return fail(MOE_ERR_INVALID_ARG, "layer or out is NULL");
  *out = nullptr;
  if (T < 1 || T > L->cfg.max_tokens) return fail(MOE_ERR_INVALID_ARG, "T out of range [1, max_tokens]");
  if (!x || !y) return fail(MOE_ERR_INVALID_ARG, "x or y is NULL");
  if (!stream) return fail(MOE_ERR_INVALID_ARG, "graph capture needs a created (non-default) stream");
  if (L->n_resident != L->cfg.n_experts)
    return fail(MOE_ERR_INVALID_ARG, "graph capture needs every expert resident (a staged forward reads the "
                                     "routing counts on the host)");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  cudaStream_t s = (cudaStream_t)stream;
  const bool prof = L->prof;
  const moe_stats_t st0 = L->st;
  L->prof = false;
  CUDA_TRY(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
  const moe_status_t r = moe_forward(L, x, T, y, stream, nullptr);
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(s, &g);
  L->prof = prof;
  const uint64_t launches = L->st.launches - st0.launches;
  L->st = st0;                                   // nothing ran yet
  if (r != MOE_OK) {
    if (g) cudaGraphDestroy(g);
    (void)cudaGetLastError();
    return r;
  }
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("graph capture failed: ") + cudaGetErrorString(e));
  cudaGraphExec_t ex = nullptr;
  const cudaError_t ei = cudaGraphInstantiate(&ex, g, 0);
  if (ei != cudaSuccess) {
    cudaGraphDestroy(g);
    return fail(MOE_ERR_CUDA, std::string("graph instantiation failed: ") + cudaGetErrorString(ei));
  }
  moe_graph *G = new (std::nothrow) moe_graph;
  if (!G) {
    cudaGraphExecDestroy(ex);
    cudaGraphDestroy(g);
    return fail(MOE_ERR_OOM, "graph handle allocation failed");
  }
  G->L = L;
  G->graph = g;
  G->exec = ex;
  G->table_version = L->table_version;
  G->launches = launches;
  *out = G;
  return MOE_OK;
}

moe_status_t moe_graph_launch(moe_graph_t G, void *stream) {
  if (!G || !G->L) return fail(MOE_ERR_INVALID_ARG, "graph is NULL");
  moe_layer *L = G->L;
  if (L->table_version != G->table_version)
    return fail(MOE_ERR_INVALID_ARG, "the slot table changed since the graph was captured");
  if (*(volatile int *)L->h_err != 0) return report_device_error(L, stream);
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  CUDA_TRY(cudaGraphLaunch(G->exec, (cudaStream_t)stream));
  L->st.forwards += 1;
  L->st.launches += G->launches;
  return MOE_OK;
}

moe_status_t moe_graph_destroy(moe_graph_t G) {
  if (!G) return MOE_OK;
  if (G->L) cudaSetDevice(G->L->cfg.device);
  if (G->exec) cudaGraphExecDestroy(G->exec);
  if (G->graph) cudaGraphDestroy(G->graph);
  delete G;
  return MOE_OK;
}

moe_status_t moe_set_policy(moe_layer_t L, int32_t policy, int32_t n_pinned, void *stream) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  if (policy < MOE_POLICY_STATIC || policy > MOE_POLICY_HYBRID) return fail(MOE_ERR_INVALID_ARG, "unknown policy");
  const int S = L->cfg.n_slots;
  if (policy == MOE_POLICY_HYBRID && (n_pinned < 0 || n_pinned > S))
    return fail(MOE_ERR_INVALID_ARG, "n_pinned must be in 0..n_slots");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  cudaStream_t st = (cudaStream_t)stream;
  CUDA_TRY(cudaStreamSynchronize(st));
  CUDA_TRY(cudaStreamSynchronize(L->side));
  if (policy == MOE_POLICY_NONE) {
    std::vector<int32_t> none(L->cfg.n_experts, -1);
    ST_TRY(moe_set_slot_table(L, none.data(), stream));
  }
  L->policy = policy;
  L->n_pinned = policy == MOE_POLICY_HYBRID ? n_pinned : 0;
  L->st.policy = policy;
  return MOE_OK;
}

moe_status_t moe_prefetch(moe_layer_t L, const int32_t *experts, int32_t n, void *stream) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  if (L->policy != MOE_POLICY_CACHE && L->policy != MOE_POLICY_HYBRID)
    return fail(MOE_ERR_INVALID_ARG, "moe_prefetch needs the CACHE or HYBRID policy");
  if (n < 0 || (n > 0 && !experts)) return fail(MOE_ERR_INVALID_ARG, "bad expert list");
  const int E = L->cfg.n_experts;
  for (int i = 0; i < n; ++i)
    if (experts[i] < 0 || experts[i] >= E) return fail(MOE_ERR_INVALID_ARG, "expert id out of range");
  if (n == 0) return MOE_OK;
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  cudaStream_t st = (cudaStream_t)stream;
  // listed experts are not evicted for one another
  std::vector<char> busy(E, 0);
  for (int i = 0; i < n; ++i) busy[experts[i]] = 1;
  const std::vector<int> cand = evictable_slots(L, busy);
  // the copies start after the work queued on `stream` (a forward in flight
  // may still read the slots they overwrite) and run on the side stream
  CUDA_TRY(cudaEventRecord(L->ev_prefetch, st));
  CUDA_TRY(cudaStreamWaitEvent(L->side, L->ev_prefetch, 0));
  const size_t bytes = L->L.bytes;
  size_t c = 0;
  int copied = 0;
  for (int i = 0; i < n && c < cand.size(); ++i) {
    const int e = experts[i];
    if (L->slot_of[e] >= 0) continue;                // resident already (or listed twice)
    const int v = cand[c++];
    CUDA_TRY(cudaMemcpyAsync(L->slots + (size_t)v * bytes, L->store + (size_t)e * bytes, bytes,
                             cudaMemcpyHostToDevice, L->side));
    const int old = L->expert_of_slot[v];
    if (old >= 0) L->slot_of[old] = -1;
    L->slot_of[e] = v;
    L->expert_of_slot[v] = e;
    ++copied;
  }
  if (copied) {
    ST_TRY(push_table(L, L->side));
    CUDA_TRY(cudaEventRecord(L->ev_prefetch, L->side));
    L->prefetch_pending = true;
    L->st.prefetched += copied;
  }
  return MOE_OK;
}

moe_status_t moe_get_stats(moe_layer_t L, moe_stats_t *out) {
  if (!L || !out) return fail(MOE_ERR_INVALID_ARG, "layer or out is NULL");
  *out = L->st;
  out->device_error = L->h_err ? *(volatile int *)L->h_err : 0;
  return MOE_OK;
}

static moe_status_t drain_profile(moe_layer *L) {
  for (auto &p : L->pend) {
    CUDA_TRY(cudaEventSynchronize(p.b));
    float ms = 0.0f;
    CUDA_TRY(cudaEventElapsedTime(&ms, p.a, p.b));
    L->prof_acc.ms[p.stage] += ms;
    L->evpool.push_back(p.a);
    L->evpool.push_back(p.b);
  }
  L->pend.clear();
  return MOE_OK;
}

moe_status_t moe_profile_enable(moe_layer_t L, int32_t enable) {
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  ST_TRY(drain_profile(L));
  L->prof_acc = moe_profile_t{};
  L->prof = enable != 0;
  return MOE_OK;
}

moe_status_t moe_profile_read(moe_layer_t L, moe_profile_t *out) {
  if (!L || !out) return fail(MOE_ERR_INVALID_ARG, "layer or out is NULL");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  ST_TRY(drain_profile(L));
  *out = L->prof_acc;
  return MOE_OK;
}

moe_status_t moe_debug_read(moe_layer_t L, int32_t which, void *dst, uint64_t bytes) {
  if (!L || !dst) return fail(MOE_ERR_INVALID_ARG, "layer or dst is NULL");
  const void *src = nullptr;
  switch (which) {
    case 1: src = L->xq; break;
    case 2: src = L->xsf; break;
    case 3: src = L->h32; break;
    case 4: src = L->hq; break;
    case 5: src = L->hsf; break;
    case 6: src = L->n_prows; break;
    case 7: src = L->prow_token; break;
    case 8: src = L->prow_pair; break;
    case 11: src = L->oprime; break;
    case 12: src = L->txq; break;
    case 13: src = L->txsf; break;
    case 14: src = L->thq; break;
    case 15: src = L->thsf; break;
    case 16: src = L->tiles; break;
    case 17: src = L->n_tiles; break;
    default: break;
  }
  if (!src) return fail(MOE_ERR_INVALID_ARG, "unknown or absent debug buffer");
  CUDA_TRY(cudaSetDevice(L->cfg.device));
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost));
  return MOE_OK;
}

void moe_destroy(moe_layer_t L) { free_layer(L); }

moe_status_t moe_debug_inject(moe_layer_t L, int32_t what) {
  if (what < 0 || what > 3) return fail(MOE_ERR_INVALID_ARG, "unknown injection");
  if (what == 2 || (!L && what == 0)) {
    g_inject_create = what;
    return MOE_OK;
  }
  if (!L) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  L->inject = what;
  return MOE_OK;
}

}  // extern "C"
