// C-ABI entry points and the host-side orchestration of a decode forward.
//
// A forward is: embedding gather -> per layer [QKV GEMM (+1/rms, RoPE, paged KV write),
// attention, O GEMM (+residual), gate/up GEMM (+1/rms, SwiGLU), down GEMM (+residual)] ->
// LM-head GEMM (+argmax/confidence partials) -> finalize (mode state update).  All kernels are
// launched with programmatic dependent launch and each decode call is replayed from a CUDA
// graph captured on first use, so the host crosses into the GPU once per call and lengths,
// positions and tokens are read by the kernels from device memory (no host sync).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <atomic>
#include <functional>
#include <string>
#include <tuple>
#include <vector>

#include "nld_internal.h"

using namespace nld;

namespace nld {
size_t attn_mma_smem_bytes(int NW, bool hilo, int stages);
size_t attn_tc_smem_bytes(bool hilo, int rt);
int attn_mma_max_clusters(int S, int NW, bool hilo, int stages, int sms, int tc);
cudaError_t init_kernel_attributes();
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 tensor map over a row-major [rows, inner] matrix, box [64 elements, box_rows],
// 128-byte swizzle, zero fill out of bounds.
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                   uint32_t box_rows) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over a pre-tiled weight matrix: a 2D view [row_tiles * (K/64) * 128 rows, 64
// elements] whose box {64, 128} is one contiguous 16 KB block.
bool make_map_tiled(CUtensorMap* map, const void* base, int n_rows, int K) {
  const uint64_t row_tiles = (n_rows + kTileRows - 1) / kTileRows;
  return make_map_bf16(map, base, kTileK, row_tiles * (K / kTileK) * kTileRows, kTileRows);
}

enum XBuf { XB_HB = 0, XB_ATTN = 1, XB_U = 2, XB_ATTZ = 3 };
// GW_OL: the O projection of a drafter forward with the adapter folded in ([W_o | B] over
// [att ; scale * A att], bf16 configuration)
enum GemmWhich { GW_QKV = 0, GW_O = 1, GW_GU = 2, GW_D = 3, GW_LM = 4, GW_OL = 5 };
enum LmKind { LM_NONE = 0, LM_ARGMAX = 1, LM_LOGITS = 2 };

std::string g_static_err;

}  // namespace

struct nld_ctx {
  nld_config c{};
  cudaStream_t stream = nullptr;
  bool own_stream = false;
  int dev = 0, sms = 148;
  bool bf16 = true;
  size_t el = 2;
  int qd = 0, kvd = 0, qkv_rows = 0, gu_rows = 0, pps = 0, n_pages = 0, kv_cap = 0, M_max = 0;
  int prefill_tokens = 2048;
  std::vector<void*> allocs;
  // weights (repacked)
  void* embed = nullptr;
  std::vector<void*> wqkv, wo, wgu, wd;
  void* wlm = nullptr;
  bool weights_ready = false;
  // LoRA drafter (optional): per layer A [r, qd] and B [d, r]; fp32 z partials
  int lora_r = 0, lora_r_alloc = 0;
  float lora_scale = 0.f;
  std::vector<void*> lora_A, lora_B;
  float* lora_zp = nullptr;
  // folded adapter (bf16): attention output rows with r_pad more columns for z = scale A att,
  // [W_o | B] per layer (pre-tiled, K = qd + r_pad), block counters of the z kernel
  int lora_rpad = 0;
  void* attz = nullptr;
  std::vector<void*> wol;
  int* lora_cnt = nullptr;
  // KV cache
  void* pool = nullptr;
  int* page_table = nullptr;
  size_t layer_elems = 0;
  // device state
  int *lens = nullptr, *pending = nullptr, *draft = nullptr, *verify = nullptr, *blk = nullptr;
  int *incomplete = nullptr, *err = nullptr, *prompt = nullptr;
  int* plens = nullptr;      // prompt length of each sequence (ragged prefill)
  int* fillnext = nullptr;   // per-sequence diffusion: block complete, causal fill due next step
  // activations
  float* h = nullptr;
  void* hb = nullptr;
  float* ssq = nullptr;
  void* qbuf = nullptr;
  void* attn = nullptr;
  void* ubuf = nullptr;
  LmPart* lm_part = nullptr;
  int lm_tiles = 0;
  float2* rope = nullptr;
  int max_clusters[9] = {0};
  unsigned* bars = nullptr;   // chain phase-boundary counters: (1 + n_layers) x kMaxPhases
  int n_bars = 0;
  int* h_pinned = nullptr;  // host: [0] error word, [1] incomplete, [2..2+B) lens, then fillnext
  // tensor maps
  std::vector<CUtensorMap> tmWqkv, tmWo, tmWgu, tmWd;
  CUtensorMap tmWlm{};
  CUtensorMap tmKV{};
  std::map<std::tuple<int, int, int>, std::pair<CUtensorMap, int>> tmX;   // (buffer, rows, kps) -> map, 3D
  int chain_x3d = 1;   // activation loads of a stage as one 3D box (0: per k-tile 2D boxes)
  int attn_rows_cap = 0;     // attention planning (profiling hook): query rows per CTA at most
  int attn_min_tiles = 0;    // and KV tiles per split at least (0: the planner's choice)
  // graphs: one per (call, batch, output pointers), at most kMaxGraphs (least recently used
  // evicted); tick = the call count at each graph's last replay
  struct GraphEntry {
    cudaGraphExec_t exec;
    unsigned long long tick;
  };
  std::map<std::vector<uintptr_t>, GraphEntry> graphs;
  unsigned long long graph_tick = 0;
  // chain tuning (profiling hook): stage cap (0 = as many as fit), k-tiles per stage
  int chain_stage_cap = 0;
  int chain_kps = 0;   // k-tiles per stage (0 = the planner's choice)
  int chain_boundary_pf = 16;   // weight boxes prefetched into L2 per CTA at a phase boundary
  int chain_pf_stages = 0;      // L2 run-ahead distance in stages (0 = off)
  int chain_warm_next = 0;      // boxes of the next chain's second phase each CTA warms in L2
  int trace_layer = -1;        // profiling hook: the layer whose attention and chain launches
  unsigned long long* attn_trace = nullptr;   // write timestamps (or -1 / null: off)
  size_t attn_trace_n = 0;
  unsigned long long* chain_trace = nullptr;
  // host-side sequence bookkeeping
  int batch = 0;
  bool started = false;
  bool verify_fresh = false;
  bool fill_pending = false;   // a complete diffusion block whose causal KV fill is deferred
  bool nl_active = false;      // per-sequence diffusion ran: fills may be due on the device
  bool quad_ready = false;     // the drafts on the device came from the last quadratic round
  long long len_upper = 0;
  uint64_t timeout_ns = 2000000000ull;
  std::string msg;
};

// SMs of the current device.
static int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  return n;
}

namespace {

nld_status fail(nld_ctx* x, nld_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (x) x->msg = buf;
  else g_static_err = buf;
  return s;
}

#define CK(call)                                                                        \
  do {                                                                                  \
    cudaError_t e_ = (call);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(x, NLD_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                  __FILE__, __LINE__);                                                  \
  } while (0)

template <typename P>
nld_status dalloc(nld_ctx* x, P** p, size_t bytes) {
  void* q = nullptr;
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(&q, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(x, NLD_ERR_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  }
  x->allocs.push_back(q);
  *p = static_cast<P*>(q);
  return NLD_OK;
}

#define TRY(expr)                \
  do {                           \
    nld_status s_ = (expr);      \
    if (s_ != NLD_OK) return s_; \
  } while (0)

nld_status validate(const nld_config* c, std::string& why) {
  char b[256];
  auto bad = [&](const char* m) {
    why = m;
    return NLD_ERR_ARG;
  };
  if (!c) return bad("config is NULL");
  if (c->n_layers < 1 || c->d_model < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 ||
      c->vocab < 2 || c->ffn_dim < 1 || c->max_batch < 1 || c->max_seq < 2)
    return bad("non-positive dimension");
  if (c->dtype != NLD_F32 && c->dtype != NLD_BF16) return bad("dtype must be NLD_F32 or NLD_BF16");
  if (c->head_dim != 64 && c->head_dim != 128) return bad("head_dim must be 64 or 128");
  if (c->dtype == NLD_BF16 && c->head_dim != 128) return bad("bf16 requires head_dim 128");
  if (c->n_q_heads % c->n_kv_heads) return bad("n_q_heads must be a multiple of n_kv_heads");
  if (c->d_model % 128) return bad("d_model must be a multiple of 128");
  if (c->ffn_dim % 64) return bad("ffn_dim must be a multiple of 64");
  if ((c->n_q_heads * c->head_dim) % 128) return bad("n_q_heads*head_dim must be a multiple of 128");
  if ((c->n_kv_heads * c->head_dim) % 64) return bad("n_kv_heads*head_dim must be a multiple of 64");
  if (c->page_size != kPage) return bad("page_size must be 64");
  if (c->block_k < 1 || c->block_k > 32) return bad("block_k must be in 1..32");
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return bad("rms_eps > 0 and rope_theta > 1 required");
  if (c->max_batch * (c->block_k + 1) > 65536) return bad("max_batch*(block_k+1) too large");
  if (c->dtype == NLD_F32 && c->max_seq > 8192)
    return bad("fp32 attention keeps a row of scores in shared memory: max_seq <= 8192");
  (void)b;
  return NLD_OK;
}

// ------------------------------------------------------------------------- GEMM dispatch --
// One projection of a chain: which weight, which layer, and its epilogue arguments.
struct ProjRef {
  int which, layer;
  EpiArgs e;
};

// 3D bf16 tensor map over a row-major [rows, inner] matrix seen as [inner/64 blocks][rows][64]
// (strides: a row inner*2 bytes, a block 128 bytes), box {64, box_rows, box_blocks}, 128-byte
// swizzle: one load brings box_blocks consecutive 64-column k-tiles of box_rows rows, stored one
// after the other ([block][row][64]), each as a 2D box would store it.
bool make_map_act3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows,
                    uint32_t box_blocks) {
  EncodeTiledFn enc = get_encoder();
  if (!enc || inner % 64) return false;
  cuuint64_t dims[3] = {64, rows, inner / 64};
  cuuint64_t strides[2] = {inner * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map of an activation buffer for loads of `rows` rows x `kps` k-tiles: the 3D form (one
// load per stage) when the encoder accepts it, else the 2D form; *is3d tells which.
const CUtensorMap* xmap(nld_ctx* x, int buf, int rows, int kps, int* is3d) {
  auto key = std::make_tuple(buf, rows, kps);
  auto it = x->tmX.find(key);
  if (it != x->tmX.end()) {
    *is3d = it->second.second;
    return &it->second.first;
  }
  CUtensorMap m;
  const void* base = buf == XB_HB ? x->hb : (buf == XB_ATTN ? x->attn : (buf == XB_ATTZ ? x->attz : x->ubuf));
  const int inner = buf == XB_HB ? x->c.d_model
                                 : (buf == XB_ATTN ? x->qd : (buf == XB_ATTZ ? x->qd + x->lora_rpad : x->c.ffn_dim));
  // bf16 activations are (hi, lo) row pairs: 2 M_max rows
  int d3 = 0;
  if (x->chain_x3d && make_map_act3d(&m, base, inner, 2ull * x->M_max, rows, kps)) {
    d3 = 1;
  } else if (!make_map_bf16(&m, base, inner, 2ull * x->M_max, rows)) {
    return nullptr;
  }
  auto& slot = x->tmX[key];
  slot = std::make_pair(m, d3);
  *is3d = d3;
  return &slot.first;
}

// Weight matrix, its tensor map and shape of projection `which` of `layer`.
struct WInfo {
  int n_rows, K, buf;
  const void* W;
  const CUtensorMap* map;
};
WInfo winfo(nld_ctx* x, int which, int layer) {
  WInfo w{};
  switch (which) {
    case GW_QKV: w = {x->qkv_rows, x->c.d_model, XB_HB, x->wqkv[layer], x->bf16 ? &x->tmWqkv[layer] : nullptr}; break;
    case GW_O: w = {x->c.d_model, x->qd, XB_ATTN, x->wo[layer], x->bf16 ? &x->tmWo[layer] : nullptr}; break;
    case GW_GU: w = {x->gu_rows, x->c.d_model, XB_HB, x->wgu[layer], x->bf16 ? &x->tmWgu[layer] : nullptr}; break;
    case GW_D: w = {x->c.d_model, x->c.ffn_dim, XB_U, x->wd[layer], x->bf16 ? &x->tmWd[layer] : nullptr}; break;
    case GW_OL: w = {x->c.d_model, x->qd + x->lora_rpad, XB_ATTZ, x->wol[layer], &x->tmWo[layer]}; break;
    default: w = {x->c.vocab, x->c.d_model, XB_HB, x->wlm, x->bf16 ? &x->tmWlm : nullptr}; break;
  }
  return w;
}

// Plan a chain of projections over M token rows.  Token columns: tiles of <= 256 (NT).  Cluster
// size CS: 4 for multi-phase decode chains (NT <= 64, where the fp32 staging buffers fit), for
// a single projection the best of 1, 2, 4, 8; 1 when NT > 64.  Per phase the K split s (a
// divisor of CS) minimises waves x (k-iterations per tile + the cross-rank handoff of a split
// tile, which measures at about six k-iterations) over the clusters that can be resident.
ChainArgs plan_chain_shapes(const int* max_clusters, const int* n_rows, const int* K, int nph, int M,
                            int hilo, int* grid_out, int stage_cap = 0, int kps_force = 0) {
  ChainArgs best{};
  long long best_cost = -1;
  int best_grid = 0;
  // with hi/lo activation rows a token takes two MMA columns: at most 128 tokens per tile
  const int max_tok = hilo ? kMaxNT / 2 : kMaxNT;
  const int tok_tiles = (M + max_tok - 1) / max_tok;
  const int per = (M + tok_tiles - 1) / tok_tiles;
  const int NT = std::max(16, (per + 15) / 16 * 16);
  int cands[4] = {1, 2, 4, 8};
  int ncand = 4;
  if (NT > 64) {
    ncand = 1;
  } else if (nph > 1) {
    cands[0] = 4;
    ncand = 1;
  }
  for (int ci = 0; ci < ncand; ++ci) {
    const int CS = cands[ci];
    const int C = max_clusters[CS];
    if (C < 1) continue;
    ChainArgs A{};
    A.nph = nph;
    A.CS = CS;
    A.NT = NT;
    long long total = 0;
    int need_clusters = 1;
    for (int p = 0; p < nph; ++p) {
      PhaseArgs& P = A.ph[p];
      P.tok_tiles = tok_tiles;
      P.row_tiles = (n_rows[p] + kTileRows - 1) / kTileRows;
      P.KT = K[p] / kTileK;
      const int tiles = P.row_tiles * P.tok_tiles;
      long long pbest = -1;
      for (int sp = 1; sp <= CS; sp *= 2) {
        if (sp > P.KT) break;
        const int ks = (P.KT + sp - 1) / sp;
        if ((sp - 1) * ks >= P.KT) continue;
        const long long groups = static_cast<long long>(C) * (CS / sp);
        const long long waves = (tiles + groups - 1) / groups;
        const long long cost = waves * (ks + (sp > 1 ? 6 : 0));
        if (pbest < 0 || cost < pbest) {
          pbest = cost;
          P.s = sp;
          P.ks = ks;
        }
      }
      total += pbest;
      need_clusters = std::max(need_clusters, (tiles * P.s + CS - 1) / CS);
    }
    if (best_cost < 0 || total < best_cost) {
      best_cost = total;
      best = A;
      best_grid = std::min(C, need_clusters) * CS;
    }
  }
  // activations: the token tile's rows rounded up to 8 (a multiple of the 128-byte swizzle
  // atom's 8 rows), so a decode tile of 33 tokens moves 40 rows per k-tile, not NT = 48
  // (several token tiles: every tile but the last is full, so all NT rows)
  best.hilo = hilo ? 1 : 0;
  const int NN = NT << best.hilo;
  best.xr = (tok_tiles == 1) ? std::min(NN, ((M << best.hilo) + 7) / 8 * 8) : NN;
  // two k-tiles (32 KB of weights) per stage: the producer/MMA barrier round trip, not HBM,
  // bounds a ring of 16 KB stages; as many stages as fit the shared-memory budget
  best.slots = 0;
  for (int p = 0; p < nph; ++p)
    if (best.ph[p].s > 1) {
      // (s - 1) senders x the chunks a rank owns (the owner keeps its own partial in registers)
      const int nch = NT / 16, s = best.ph[p].s;
      best.slots = std::max(best.slots, (s - 1) * ((nch + s - 1) / s));
    }
  // ring: two k-tiles (32 KB of weights) per stage, so one producer/MMA barrier round trip moves
  // 32 KB, with as many stages as fit the shared-memory budget; when wide activation boxes leave
  // room for fewer than three such stages, one k-tile per stage (more, smaller stages)
  const int st_max = stage_cap > 0 ? std::min(stage_cap, gemm_chain_max_stages()) : gemm_chain_max_stages();
  auto fit = [&](int kps) {
    for (int st = st_max; st > 2; --st)
      if (gemm_chain_smem_bytes(NT, NN, best.xr, kps, st, best.CS, best.slots) <= kChainSmemBudget) return st;
    return 2;
  };
  best.kps = (kps_force > 0) ? kps_force : 2;
  best.stages = fit(best.kps);
  if (kps_force <= 0 && best.stages < 3) {
    best.kps = 1;
    best.stages = fit(1);
  }
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * NN)) cols <<= 1;
  best.tmem_cols = cols;
  if (grid_out) *grid_out = best_grid;
  return best;
}

ChainArgs plan_chain(nld_ctx* x, const ProjRef* pr, int nph, int M, int* grid_out) {
  int nr[kMaxPhases], kd[kMaxPhases];
  for (int p = 0; p < nph; ++p) {
    const WInfo w = winfo(x, pr[p].which, pr[p].layer);
    nr[p] = w.n_rows;
    kd[p] = w.K;
  }
  return plan_chain_shapes(x->max_clusters, nr, kd, nph, M, x->bf16 ? 1 : 0, grid_out, x->chain_stage_cap,
                           x->chain_kps);
}

// Launch a chain of projections (the SIMT kernel one by one for the fp32 configuration).
// `bar`: this launch's phase-boundary counters.  next_*: the projection after this launch
// (L2 warm-up of its first weight boxes), or next_which < 0.
nld_status chain(nld_ctx* x, const ProjRef* pr, int nph, int M, bool pdl, unsigned* bar,
                 const ProjRef* next_pr, int next_nph, unsigned long long* trace = nullptr) {
  if (!x->bf16) {
    for (int p = 0; p < nph; ++p) {
      const WInfo w = winfo(x, pr[p].which, pr[p].layer);
      EpiArgs e = pr[p].e;
      e.n_rows = w.n_rows;
      const void* X = w.buf == XB_HB ? x->hb : (w.buf == XB_ATTN ? x->attn : x->ubuf);
      CK(launch_gemm_simt(x->stream, static_cast<const float*>(w.W), static_cast<const float*>(X),
                          w.n_rows, w.K, M, e, pdl));
    }
    return NLD_OK;
  }
  int grid = 0;
  ChainArgs A = plan_chain(x, pr, nph, M, &grid);
  for (int p = 0; p < nph; ++p) {
    const WInfo w = winfo(x, pr[p].which, pr[p].layer);
    A.ph[p].tmW = *w.map;
    A.ph[p].W = w.W;
    int is3d = 0;
    const CUtensorMap* tmX = xmap(x, w.buf, A.xr, A.kps, &is3d);
    if (!tmX) return fail(x, NLD_ERR_CUDA, "tensor map encode failed (activation buffer)");
    A.ph[p].tmX = *tmX;
    A.ph[p].x3d = is3d;
    A.ph[p].e = pr[p].e;
    A.ph[p].e.n_rows = w.n_rows;
  }
  A.bar = bar;
  A.trace = trace;
  A.boundary_pf = x->chain_boundary_pf;
  A.pf_stages = x->chain_pf_stages;
  if (next_pr && next_nph > 0) {
    int ngrid = 0;
    const ChainArgs N = plan_chain(x, next_pr, next_nph, M, &ngrid);
    A.next_valid = 1;
    A.next_CS = N.CS;
    A.next_grid = ngrid;
    for (int j = 0; j < 2 && j < next_nph; ++j) {
      WarmPhase& wp = A.next[j];
      wp.W = winfo(x, next_pr[j].which, next_pr[j].layer).W;
      wp.s = N.ph[j].s;
      wp.tok_tiles = N.ph[j].tok_tiles;
      wp.ks = N.ph[j].ks;
      wp.KT = N.ph[j].KT;
      wp.tiles = N.ph[j].row_tiles * N.ph[j].tok_tiles;
      wp.boxes = j == 0 ? N.stages * N.kps + 8 : x->chain_warm_next;
    }
  }
  CK(launch_gemm_chain(x->stream, A, grid, x->timeout_ns, pdl));
  return NLD_OK;
}

// Clusters of S attention CTAs (NW warps, `stages` ring stages; or the tcgen05 kernel) resident
// at once.
using AttnCapacity = std::function<int(int S, int NW, int stages, int tc)>;

// Which kernel serves the tensor-core attention (profiling hook): 0 the planner's choice,
// 1 tcgen05, 2 mma.sync, 3 / 4 tcgen05 with 2 / 4 softmax threads per row.
std::atomic<int> g_attn_kernel{0};
// Keys per KV tile of the tcgen05 kernel (profiling and test hook): 0 the planner's choice, 64
// or 128.
std::atomic<int> g_attn_tile{0};

// rows_cap: query rows (positions x heads) per CTA at most (16..144: 9 warps); min_tiles: KV
// tiles a split takes at least; 0 = the planner's choice for either.  tile: keys per tcgen05 KV
// tile, 0 = the planner's choice.  hilo: q and P as (hi, lo) operand pairs (the model's
// forwards) rather than bf16 q (the stand-alone call).
void attn_plan(int batch, int m, int Hq, int Hkv, int max_len, int sms, AttnArgs& a, const AttnCapacity& cap,
               int rows_cap = 0, int min_tiles = 0, int kernel = 0, int tile = 0, bool hilo = true) {
  a.G = Hq / Hkv;
  const int n_tiles = std::max(1, (max_len + kPage - 1) / kPage);
  auto q_tiles_for = [&](int c) {
    const int qt_max = std::min(m, std::max(1, c / a.G));
    return (m + qt_max - 1) / qt_max;
  };
  // Latency regime (a few sequences): even split 8 ways, whole query tiles would leave most SMs
  // idle, so the query positions are cut into tiles of <= 64 rows (one warp per SM
  // sub-partition: a KV tile then costs a quarter of the MMA time of an 8-warp CTA), the keys
  // into splits of single tiles, and the ring holds 2 stages (about 100 KB, two CTAs per SM).
  // Otherwise tiles of up to 144 rows (a 33-position verify block of 4 heads in one 9-warp
  // CTA) read each K/V tile once for as many query rows as possible, through a 3-stage ring.
  // The tcgen05 kernel takes query tiles of up to 128 rows (one MMA tile, in either regime),
  // and a KV tile costs it about what a 56-row tile costs mma.sync, whatever its rows (mma.sync
  // scales with the rows).  So it serves tiles of >= 64 rows in the latency regime and, with
  // many sequences, where its query tiles x 56 stay below the rows of mma.sync's tiles of up to
  // 144 (a 16-position block of 4 heads: 56 < 64; a 33-position one in two tiles: 112 < 132),
  // unless an explicit tile above 128 rows is asked for.
  const bool latency = batch * Hkv * q_tiles_for(144) * 8 < 2 * sms;
  const int tc_rows = ((m + q_tiles_for(128) - 1) / q_tiles_for(128)) * a.G;
  const int mma_rows = ((m + q_tiles_for(144) - 1) / q_tiles_for(144)) * a.G;
  const bool use_tc = kernel == 1 || kernel >= 3 ||
                      (kernel == 0 && rows_cap <= 128 &&
                       (latency ? tc_rows >= 64 : q_tiles_for(128) * 56 < q_tiles_for(144) * mma_rows));
  // softmax threads per row (set below for the planner's choice)
  int tc = !use_tc ? 0 : kernel == 3 ? 2 : 4;
  if (rows_cap <= 0) rows_cap = tc ? 128 : (latency ? 64 : 144);
  if (tc) rows_cap = std::min(rows_cap, 128);
  if (min_tiles <= 0) min_tiles = latency ? 1 : 2;
  a.min_tiles = min_tiles;
  a.stages = (latency || tc) ? 2 : 3;
  a.tc = tc;
  // query positions per CTA: as many as rows_cap allows, spread evenly over the query tiles
  const int nq = q_tiles_for(rows_cap);
  a.QT = (m + nq - 1) / nq;
  a.q_tiles = (m + a.QT - 1) / a.QT;
  a.rows = a.QT * a.G;
  a.NW = (a.rows + 15) / 16;
  // KV splits of one (sequence, kv head, query tile) form a cluster of at most 8 CTAs.  Split
  // only while the grid is short of two CTAs per SM, keep >= min_tiles KV tiles per split, take
  // no more splits than lets every cluster be resident at once (a second wave doubles the
  // latency), and launch no split that the tiles per split leave empty.
  // The tcgen05 kernel's KV tiles: 64 keys where a split holds up to 3 pages (a chain of one to
  // three short tiles is the latency: the batch-1 round at short prefixes), 128 where splits are
  // longer (S with N = 128: half the S MMAs per key); its splits are counted in those tiles
  // (measured: 64 win at <= 2 pages per split, even at 3, 128 win from 4 by 0.5-5 %).
  const int units = batch * a.q_tiles * Hkv;
  auto split_plan = [&](int pg, int* per_pages) {
    const int kt = (n_tiles + pg - 1) / pg;                       // KV tiles of the kernel
    const int min_kt = (min_tiles + pg - 1) / pg;
    int S = 1;
    if (units < 2 * sms) {
      int s_max = std::max(1, std::min({8, (2 * sms + units - 1) / units, std::max(1, kt / min_kt)}));
      while (s_max > 1 && units > cap(s_max, a.NW, a.stages, tc)) --s_max;
      const int per = std::max(min_kt, (kt + s_max - 1) / s_max);
      S = std::max(1, (kt + per - 1) / per);
    }
    *per_pages = std::max(min_kt, (kt + S - 1) / S) * pg;
    return S;
  };
  int per_pages = 0;
  a.S = split_plan(1, &per_pages);
  a.tc_tile = 64;
  if (use_tc && (tile == 128 || (tile == 0 && per_pages > 3))) {
    a.tc_tile = 128;
    a.S = split_plan(2, &per_pages);
  }
  // tcgen05 softmax threads per row: 4 (16 warps) shorten a CTA's fixed costs and each KV tile's
  // latency chain, which short splits wait on; 2 (8 warps) issue fewer instructions per tile,
  // which long splits are bound by (measured: 4 win at <= 17 pages per CTA by up to 20 %, 2 at
  // 65 and 257 pages by 5-8 %, even at 33).  With bf16 q (half the MMAs and P stores of a
  // tile) and at most half the SMs busy, 2 win from 8 pages (4k keys at batch 1: 18.6 vs 20.4
  // us); the model's (hi, lo) forwards keep 4 there (14B round at a 4k prefix: 4 win by 4 %).
  if (use_tc && (kernel == 0 || kernel == 1)) {
    tc = per_pages > 32 ? 2 : 4;
    if (!hilo && per_pages >= 8 && 2 * units * a.S <= sms) tc = 2;
    a.tc = tc;
  }
}

// The device's cluster capacity for the attention kernel (occupancy query, cached).
int attn_device_capacity(bool hilo, int S, int NW, int stages, int tc) {
  static int cache[16][9][10][2][4][3];   // [device][S][NW][hilo][stages][tc / 2]; 0 = not yet queried
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 16 || S < 1 || S > 8 || NW < 1 || NW > 9 || stages < 2 ||
      stages > 3 || (tc != 0 && tc != 2 && tc != 4)) {
    cudaGetLastError();
    return 1;
  }
  static std::mutex mu;   // the stand-alone attention may be called from several threads
  std::lock_guard<std::mutex> lock(mu);
  int& c = cache[dev][S][NW][hilo ? 1 : 0][stages][tc / 2];
  if (c == 0) c = attn_mma_max_clusters(S, NW, hilo, stages, device_sms(), tc);
  return c;
}

EpiArgs base_epi(nld_ctx* x, int M, int m) {
  EpiArgs e{};
  e.M = M;
  e.m = m;
  e.ssq_in = x->ssq;
  e.ssq_tiles = x->c.d_model / kTileRows;
  e.ssq_ld = x->M_max;
  e.inv_d = 1.0f / static_cast<float>(x->c.d_model);
  e.eps = x->c.rms_eps;
  e.Hq = x->c.n_q_heads;
  e.Hkv = x->c.n_kv_heads;
  e.hd = x->c.head_dim;
  e.page_table = x->page_table;
  e.pps = x->pps;
  e.lens = x->lens;
  e.rope = x->rope;
  e.kv_cap = x->kv_cap;
  e.h = x->h;
  e.hb = x->hb;
  e.ssq_out = x->ssq;
  e.d = x->c.d_model;
  e.u_out = x->ubuf;
  e.F = x->c.ffn_dim;
  e.lm_part = x->lm_part;
  e.lm_tiles = x->lm_tiles;
  e.V = x->c.vocab;
  e.q_out = x->qbuf;
  e.hilo = x->bf16 ? 1 : 0;
  e.err = x->err;
  return e;
}

struct FwdSpec {
  int mode;          // FwdMode of the embedding / finalize
  int B, m, bs;      // sequences, rows per sequence, attention block size
  int lm;            // LmKind
  float* logits;     // LM_LOGITS target
  int chunk0;        // prefill: first prompt position of this chunk
  int prompt_len;
  bool last_chunk;
  int causal_rows;   // attention: leading strictly causal rows (fused diffusion fill)
  const int* causal_seq;   // per-sequence diffusion: sequences whose rows are all causal
  int quad_k;        // quadratic self-speculation forward with block k (0 = off)
};

// Launch one forward (no finalize).
nld_status launch_forward(nld_ctx* x, const FwdSpec& f) {
  const int M = f.B * f.m;
  const bool pdl = true;
  EmbedArgs ea{};
  ea.E = x->embed;
  ea.d = x->c.d_model;
  ea.V = x->c.vocab;
  ea.m = f.m;
  ea.mode = f.mode;
  ea.k = x->c.block_k;
  ea.pending = x->pending;
  ea.draft = x->draft;
  ea.blk = x->blk;
  ea.prompt = x->prompt;
  ea.prompt_len = f.prompt_len;
  ea.chunk0 = f.chunk0;
  ea.plens = (f.mode == FWD_PREFILL) ? x->plens : nullptr;
  ea.lens = x->lens;
  ea.h = x->h;
  ea.hb = x->hb;
  ea.ssq = x->ssq;
  ea.ssq_ld = x->M_max;
  ea.hilo = x->bf16 ? 1 : 0;
  ea.err = x->err;
  CK(launch_embed(x->stream, ea, M, x->bf16, pdl));

  const int max_len = static_cast<int>(std::min<long long>(x->kv_cap, x->len_upper + f.m));
  AttnArgs aa{};
  bool attn_traced = false;
  aa.q = x->qbuf;
  // drafter forwards of a context with an adapter: on the tensor-core path the adapter is folded
  // into the O projection; the attention writes rows with room for z
  const bool lora_fwd = x->lora_r > 0 && (f.mode == FWD_DRAFT || f.mode == FWD_DIFFUSE || f.mode == FWD_FILLDIFF ||
                                          f.mode == FWD_NLDIFF || f.mode == FWD_QUAD);
  const bool folded = lora_fwd && x->bf16;
  aa.out = folded ? x->attz : x->attn;
  aa.out_ld = static_cast<size_t>(x->qd) + (folded ? x->lora_rpad : 0);
  aa.m = f.m;
  aa.Hq = x->c.n_q_heads;
  aa.Hkv = x->c.n_kv_heads;
  aa.hd = x->c.head_dim;
  aa.lens = x->lens;
  aa.page_table = x->page_table;
  aa.pps = x->pps;
  aa.block_size = f.bs;
  aa.causal_rows = f.causal_rows;
  aa.causal_seq = f.causal_seq;
  aa.err = x->err;
  aa.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(x->c.head_dim)));
  aa.hilo = x->bf16 ? 1 : 0;
  aa.quad_k = f.quad_k;
  if (x->bf16) {
    attn_plan(f.B, f.m, aa.Hq, aa.Hkv, max_len, x->sms, aa,
              [](int S, int NW, int stages, int tc) { return attn_device_capacity(true, S, NW, stages, tc); },
              x->attn_rows_cap, x->attn_min_tiles, g_attn_kernel.load(), g_attn_tile.load());
    const size_t ctas = static_cast<size_t>(aa.S) * aa.Hkv * f.B * aa.q_tiles;
    attn_traced = x->attn_trace && ctas * 16 <= x->attn_trace_n;
  } else {
    aa.G = aa.Hq / aa.Hkv;
  }

  // projections: QKV(0) | per layer: attention, chain [O, gate/up, down, QKV(l+1) or, for the
  // last layer, the LM head]
  const int L = x->c.n_layers;
  auto proj = [&](int which, int layer) {
    ProjRef r{which, layer, base_epi(x, M, f.m)};
    r.e.quad_k = f.quad_k;
    static const int kinds[6] = {EPI_QKV, EPI_RESID, EPI_SWIGLU, EPI_RESID, EPI_LMHEAD, EPI_RESID};
    r.e.kind = kinds[which];
    if (which == GW_QKV)
      r.e.kv_layer = static_cast<char*>(x->pool) + static_cast<size_t>(layer) * x->layer_elems * x->el;
    if (which == GW_LM) {
      r.e.kind = (f.lm == LM_LOGITS) ? EPI_LOGITS : EPI_LMHEAD;
      r.e.logits = f.logits;
    }
    return r;
  };
  auto layer_chain = [&](int l, ProjRef* out) {
    int n = 0;
    out[n++] = proj(folded ? GW_OL : GW_O, l);
    out[n++] = proj(GW_GU, l);
    out[n++] = proj(GW_D, l);
    if (l + 1 < L) out[n++] = proj(GW_QKV, l + 1);
    return n;
  };
  ProjRef cur[kMaxPhases], nxt[kMaxPhases];
  {
    const ProjRef q0 = proj(GW_QKV, 0);
    const int nn = layer_chain(0, nxt);
    TRY(chain(x, &q0, 1, M, pdl, x->bars, nxt, nn));
  }
  for (int l = 0; l < L; ++l) {
    if (x->bf16) {
      aa.layer_row0 = l * x->n_pages * 2 * x->c.n_kv_heads * kPage;
      aa.trace = (attn_traced && l == x->trace_layer) ? x->attn_trace : nullptr;
      CK(launch_attention_mma(x->stream, &x->tmKV, aa, f.B, pdl));
    } else {
      aa.pool = static_cast<char*>(x->pool) + static_cast<size_t>(l) * x->layer_elems * x->el;
      CK(launch_attention_simt(x->stream, aa, f.B, true, x->kv_cap, pdl));
    }
    // LoRA drafter: the block-bidirectional rows (the fused fill's causal rows excluded).  Folded
    // (bf16): one launch writes z = scale * A att beside the attention output, and the chain's
    // O projection takes B as r_pad more K columns; fp32: z, then h += scale * B z
    if (folded)
      CK(launch_lora_z(x->stream, x->lora_A[l], x->attz, aa.out_ld, x->lora_zp, x->lora_cnt, x->attz, aa.out_ld,
                       M, x->qd, x->lora_r, x->lora_scale, f.m, f.causal_rows, f.causal_seq, pdl));
    else if (lora_fwd)
      CK(launch_lora(x->stream, x->lora_A[l], x->lora_B[l], x->attn, x->lora_zp, x->h, M, x->qd,
                     x->c.d_model, x->lora_r, x->lora_scale, f.m, f.causal_rows, f.causal_seq,
                     x->bf16, x->bf16, pdl));
    int n = layer_chain(l, cur);
    int nn = 0;
    if (l + 1 < L) {
      nn = layer_chain(l + 1, nxt);
    } else if (f.lm != LM_NONE) {
      // the last layer's chain ends with the final norm + LM head: its weights stream in across
      // the phase boundary instead of after a kernel boundary
      cur[n++] = proj(GW_LM, 0);
    }
    TRY(chain(x, cur, n, M, pdl, x->bars + (1 + l) * kMaxPhases, nn ? nxt : nullptr, nn,
              l == x->trace_layer ? x->chain_trace : nullptr));
  }
  return NLD_OK;
}

FinalizeArgs base_fin(nld_ctx* x, int mode, int m) {
  FinalizeArgs a{};
  a.mode = mode;
  a.m = m;
  a.k = x->c.block_k;
  a.V = x->c.vocab;
  a.lm_tiles = x->lm_tiles;
  a.lm_part = x->lm_part;
  a.lens = x->lens;
  a.pending = x->pending;
  a.draft = x->draft;
  a.verify = x->verify;
  a.blk = x->blk;
  a.incomplete = x->incomplete;
  a.prompt = nullptr;
  a.commit = 1;
  a.kv_cap = x->kv_cap;
  a.err = x->err;
  a.fillnext = x->fillnext;
  a.state_out = nullptr;
  return a;
}

nld_status finalize(nld_ctx* x, const FinalizeArgs& a) {
  CK(launch_finalize(x->stream, a, x->batch, true));
  return NLD_OK;
}

constexpr size_t kMaxGraphs = 64;

void drop_graphs(nld_ctx* x) {
  for (auto& kv : x->graphs) cudaGraphExecDestroy(kv.second.exec);
  x->graphs.clear();
}

// Capture `body` into a graph keyed by `key` on first use, then replay it.  A caller that keeps
// passing fresh output buffers makes new keys: past kMaxGraphs graphs the least recently
// replayed one is destroyed (after the stream drains, so no replay of it is in flight).
template <typename F>
nld_status run_graph(nld_ctx* x, const std::vector<uintptr_t>& key, F body) {
  auto it = x->graphs.find(key);
  if (it == x->graphs.end()) {
    if (x->graphs.size() >= kMaxGraphs) {
      auto victim = x->graphs.begin();
      for (auto g = x->graphs.begin(); g != x->graphs.end(); ++g)
        if (g->second.tick < victim->second.tick) victim = g;
      CK(cudaStreamSynchronize(x->stream));
      cudaGraphExecDestroy(victim->second.exec);
      x->graphs.erase(victim);
    }
    cudaGraph_t g = nullptr;
    CK(cudaStreamBeginCapture(x->stream, cudaStreamCaptureModeThreadLocal));
    nld_status s = body();
    cudaError_t ce = cudaStreamEndCapture(x->stream, &g);
    if (s != NLD_OK) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      return s;
    }
    if (ce != cudaSuccess) return fail(x, NLD_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ce));
    cudaGraphExec_t ex = nullptr;
    ce = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    if (ce != cudaSuccess) return fail(x, NLD_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(ce));
    it = x->graphs.emplace(key, nld_ctx::GraphEntry{ex, 0}).first;
  }
  it->second.tick = ++x->graph_tick;
  CK(cudaGraphLaunch(it->second.exec, x->stream));
  return NLD_OK;
}

// Make sure `grow` more committed rows fit; refresh the exact lengths from the device when
// the host's upper bound says they might not.
nld_status ensure_capacity(nld_ctx* x, long long grow) {
  if (x->len_upper + grow <= x->c.max_seq) return NLD_OK;
  CK(cudaMemcpyAsync(x->h_pinned + 2, x->lens, sizeof(int) * x->batch, cudaMemcpyDeviceToHost, x->stream));
  CK(cudaStreamSynchronize(x->stream));
  long long mx = 0;
  for (int b = 0; b < x->batch; ++b) mx = std::max<long long>(mx, x->h_pinned[2 + b]);
  x->len_upper = mx;
  if (x->len_upper + grow > x->c.max_seq)
    return fail(x, NLD_ERR_KV_FULL, "sequence length %lld + %lld would exceed max_seq %d", mx, grow,
                x->c.max_seq);
  return NLD_OK;
}

nld_status need_started(nld_ctx* x) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if (!x->weights_ready) return fail(x, NLD_ERR_STATE, "weights not initialised");
  if (!x->started) return fail(x, NLD_ERR_STATE, "no sequences: call nld_prefill first");
  return NLD_OK;
}

}  // namespace

// =================================================================================== API ===
extern "C" {

nld_status nld_create(const nld_config* cfg, void* cuda_stream, nld_ctx** out) {
  if (!out) return fail(nullptr, NLD_ERR_ARG, "out is NULL");
  *out = nullptr;
  std::string why;
  if (validate(cfg, why) != NLD_OK) return fail(nullptr, NLD_ERR_ARG, "invalid config: %s", why.c_str());
  nld_ctx* x = new nld_ctx();
  x->c = *cfg;
  const nld_config& c = x->c;
  auto bail = [&](nld_status s) {
    g_static_err = x->msg;
    nld_destroy(x);
    return s;
  };
  if (cudaGetDevice(&x->dev) != cudaSuccess) {
    cudaGetLastError();
    delete x;
    return fail(nullptr, NLD_ERR_CUDA, "no CUDA device");
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, x->dev) != cudaSuccess) {
    delete x;
    return fail(nullptr, NLD_ERR_CUDA, "cudaGetDeviceProperties failed");
  }
  x->sms = prop.multiProcessorCount;
  x->bf16 = (c.dtype == NLD_BF16);
  if (x->bf16 && prop.major != 10) {
    delete x;
    return fail(nullptr, NLD_ERR_UNSUPPORTED, "bf16 kernels need an sm_100 GPU (found sm_%d%d)",
                prop.major, prop.minor);
  }
  x->el = x->bf16 ? 2 : 4;
  {
    cudaError_t ae = init_kernel_attributes();
    if (ae != cudaSuccess) {
      cudaGetLastError();
      delete x;
      return fail(nullptr, NLD_ERR_CUDA, "setting kernel shared-memory limits failed: %s",
                  cudaGetErrorString(ae));
    }
  }
  if (cuda_stream) {
    x->stream = static_cast<cudaStream_t>(cuda_stream);
  } else {
    if (cudaStreamCreateWithFlags(&x->stream, cudaStreamNonBlocking) != cudaSuccess) {
      delete x;
      return fail(nullptr, NLD_ERR_CUDA, "stream creation failed");
    }
    x->own_stream = true;
  }
  x->qd = c.n_q_heads * c.head_dim;
  x->kvd = c.n_kv_heads * c.head_dim;
  x->qkv_rows = x->qd + 2 * x->kvd;
  x->gu_rows = 2 * c.ffn_dim;
  x->pps = (c.max_seq + c.block_k + 1 + kPage - 1) / kPage;
  x->kv_cap = x->pps * kPage;
  x->n_pages = c.max_batch * x->pps;
  x->prefill_tokens = 2048;
  x->M_max = std::max(c.max_batch * (c.block_k + 1), x->prefill_tokens);
  x->M_max = (x->M_max + 15) / 16 * 16;
  x->lm_tiles = (c.vocab + kTileRows - 1) / kTileRows;
  const size_t el = x->el;
  const int d = c.d_model;

  // KV pool [layer][page][2][Hkv][64][hd] and a page table that interleaves the sequences'
  // pages (page j of sequence b is physical page j*max_batch + b), so kernels never rely on
  // a sequence's pages being adjacent.
  x->layer_elems = static_cast<size_t>(x->n_pages) * 2 * c.n_kv_heads * kPage * c.head_dim;
  if (static_cast<long long>(c.n_layers) * x->n_pages * 2 * c.n_kv_heads * kPage > INT32_MAX)
    return bail(fail(x, NLD_ERR_ARG, "KV pool too large for 32-bit TMA row coordinates"));
  nld_status s;
  if ((s = dalloc(x, &x->pool, x->layer_elems * c.n_layers * el)) != NLD_OK) return bail(s);
  if (cudaMemsetAsync(x->pool, 0, x->layer_elems * c.n_layers * el, x->stream) != cudaSuccess)
    return bail(fail(x, NLD_ERR_CUDA, "pool memset failed"));
  {
    std::vector<int> pt(static_cast<size_t>(c.max_batch) * x->pps);
    for (int b = 0; b < c.max_batch; ++b)
      for (int j = 0; j < x->pps; ++j) pt[static_cast<size_t>(b) * x->pps + j] = j * c.max_batch + b;
    if ((s = dalloc(x, &x->page_table, pt.size() * sizeof(int))) != NLD_OK) return bail(s);
    if (cudaMemcpy(x->page_table, pt.data(), pt.size() * sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(x, NLD_ERR_CUDA, "page table upload failed"));
  }
  // RoPE table [kv_cap][hd/2] of (cos, sin) of pos * theta^(-2i/hd), computed in double.
  {
    const int half = c.head_dim / 2;
    std::vector<float2> tab(static_cast<size_t>(x->kv_cap) * half);
    for (int p = 0; p < x->kv_cap; ++p)
      for (int i = 0; i < half; ++i) {
        const double inv_freq = std::pow(static_cast<double>(c.rope_theta), -2.0 * i / c.head_dim);
        const double ang = static_cast<double>(p) * inv_freq;
        tab[static_cast<size_t>(p) * half + i] = make_float2(static_cast<float>(std::cos(ang)),
                                                             static_cast<float>(std::sin(ang)));
      }
    if ((s = dalloc(x, &x->rope, tab.size() * sizeof(float2))) != NLD_OK) return bail(s);
    if (cudaMemcpy(x->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess)
      return bail(fail(x, NLD_ERR_CUDA, "rope table upload failed"));
  }
  const int B = c.max_batch, k = c.block_k;
  if ((s = dalloc(x, &x->lens, B * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->pending, B * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->draft, static_cast<size_t>(B) * k * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->verify, static_cast<size_t>(B) * (k + 1) * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->blk, static_cast<size_t>(B) * k * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->incomplete, 16)) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->err, 16)) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->prompt, static_cast<size_t>(B) * c.max_seq * sizeof(int))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->plens, B * sizeof(int))) != NLD_OK) return bail(s);
  const size_t Mm = x->M_max;
  if ((s = dalloc(x, &x->h, Mm * d * sizeof(float))) != NLD_OK) return bail(s);
  // activation operands: fp32 values (fp32 path) or (hi, lo) bf16 row pairs: 4 bytes each;
  // q is fp32 in both (the bf16 attention splits it itself)
  const size_t ael = 4;
  if ((s = dalloc(x, &x->hb, Mm * d * ael)) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->ssq, (d / kTileRows) * Mm * sizeof(float))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->qbuf, Mm * x->qd * sizeof(float))) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->attn, Mm * x->qd * ael)) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->ubuf, Mm * c.ffn_dim * ael)) != NLD_OK) return bail(s);
  if ((s = dalloc(x, &x->lm_part, Mm * x->lm_tiles * sizeof(LmPart))) != NLD_OK) return bail(s);
  x->n_bars = (2 + c.n_layers) * kMaxPhases;
  if ((s = dalloc(x, &x->bars, x->n_bars * sizeof(unsigned))) != NLD_OK) return bail(s);
  if (cudaMemset(x->bars, 0, x->n_bars * sizeof(unsigned)) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  // resident clusters of each split size (one GEMM CTA per SM)
  if (x->bf16)
    for (int sp = 1; sp <= 8; ++sp) x->max_clusters[sp] = gemm_tc_max_clusters(sp, 200 * 1024, x->sms);
  if (cudaMemset(x->err, 0, 16) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMemset(x->lens, 0, B * sizeof(int)) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMemset(x->h, 0, Mm * d * sizeof(float)) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMemset(x->hb, 0, Mm * d * ael) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMemset(x->attn, 0, Mm * x->qd * ael) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMemset(x->ubuf, 0, Mm * c.ffn_dim * ael) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if ((s = dalloc(x, &x->fillnext, B * sizeof(int))) != NLD_OK) return bail(s);
  if (cudaMemset(x->fillnext, 0, B * sizeof(int)) != cudaSuccess) return bail(fail(x, NLD_ERR_CUDA, "memset"));
  if (cudaMallocHost(&x->h_pinned, (4 + 2 * B) * sizeof(int)) != cudaSuccess)
    return bail(fail(x, NLD_ERR_OOM, "pinned host allocation failed"));
  if (x->bf16) {
    const uint64_t rows = static_cast<uint64_t>(c.n_layers) * x->n_pages * 2 * c.n_kv_heads * kPage;
    if (!make_map_bf16(&x->tmKV, x->pool, c.head_dim, rows, kPage))
      return bail(fail(x, NLD_ERR_CUDA, "tensor map encode failed (KV pool)"));
  }
  if (cudaStreamSynchronize(x->stream) != cudaSuccess)
    return bail(fail(x, NLD_ERR_CUDA, "initialisation failed"));
  *out = x;
  return NLD_OK;
}

nld_status nld_destroy(nld_ctx* x) {
  if (!x) return NLD_OK;
  if (x->stream) cudaStreamSynchronize(x->stream);
  drop_graphs(x);
  for (void* p : x->allocs) cudaFree(p);
  x->allocs.clear();
  if (x->h_pinned) cudaFreeHost(x->h_pinned);
  if (x->own_stream && x->stream) cudaStreamDestroy(x->stream);
  delete x;
  return NLD_OK;
}

nld_status nld_init_lora(nld_ctx* x, int rank, float scale, const void* const* tensors, int n_tensors,
                         int on_device) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if (!x->weights_ready) return fail(x, NLD_ERR_STATE, "weights not initialised");
  const int L = x->c.n_layers, d = x->c.d_model;
  if (rank < 0 || rank > 256 || rank % 8)
    return fail(x, NLD_ERR_ARG, "LoRA rank %d: a multiple of 8 in [8, 256] (0 switches off)", rank);
  if (x->qd % 8) return fail(x, NLD_ERR_UNSUPPORTED, "LoRA needs Hq*hd a multiple of 8");
  if (!std::isfinite(scale)) return fail(x, NLD_ERR_ARG, "LoRA scale is not finite");
  if (rank > 0) {
    if (!tensors || n_tensors != 2 * L)
      return fail(x, NLD_ERR_ARG, "expected %d LoRA tensors, got %d", 2 * L, n_tensors);
    for (int i = 0; i < n_tensors; ++i)
      if (!tensors[i]) return fail(x, NLD_ERR_ARG, "LoRA tensor %d is NULL", i);
    if (!x->lora_A.empty() && rank != x->lora_r_alloc)
      return fail(x, NLD_ERR_STATE, "LoRA rank %d differs from the first load (%d)", rank, x->lora_r_alloc);
  }
  CK(cudaStreamSynchronize(x->stream));
  // the captured graphs hold the old launch sequence (or none of the LoRA launches)
  drop_graphs(x);
  x->lora_r = 0;
  if (rank == 0) return NLD_OK;
  const size_t el = x->el;
  nld_status s;
  if (x->lora_A.empty()) {
    // allocate into locals; the context takes them only when all succeeded (a failed first
    // load leaves no half-made adapter behind; what was allocated is freed with the context)
    std::vector<void*> A(L, nullptr), Bm(L, nullptr);
    float* zp = nullptr;
    for (int l = 0; l < L; ++l) {
      if ((s = dalloc(x, &A[l], static_cast<size_t>(rank) * x->qd * el)) != NLD_OK) return s;
      if ((s = dalloc(x, &Bm[l], static_cast<size_t>(d) * rank * el)) != NLD_OK) return s;
    }
    const size_t nzp = static_cast<size_t>(lora_n_ks(x->qd, x->bf16)) * x->M_max * rank;
    if ((s = dalloc(x, &zp, nzp * sizeof(float))) != NLD_OK) return s;
    x->lora_A.swap(A);
    x->lora_B.swap(Bm);
    x->lora_zp = zp;
    x->lora_r_alloc = rank;
  }
  const cudaMemcpyKind kind = on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  for (int l = 0; l < L; ++l) {
    CK(cudaMemcpyAsync(x->lora_A[l], tensors[2 * l], static_cast<size_t>(rank) * x->qd * el, kind, x->stream));
    CK(cudaMemcpyAsync(x->lora_B[l], tensors[2 * l + 1], static_cast<size_t>(d) * rank * el, kind, x->stream));
  }
  if (x->bf16) {
    // the folded adapter: [W_o | B] per layer as pre-tiled blocks (row tile, k tile), K = qd +
    // r_pad (B's columns zero-padded to a whole k tile), and the attention output buffer with
    // r_pad more columns per (hi, lo) row for z
    const int rpad = (rank + kTileK - 1) / kTileK * kTileK;
    const int KT = x->qd / kTileK, KB = rpad / kTileK, KTL = KT + KB, RT = d / kTileRows;
    const size_t blk = static_cast<size_t>(kTileRows) * kTileK * el;   // 16 KB
    if (x->wol.empty()) {
      std::vector<void*> wol(L, nullptr);
      void* attz = nullptr;
      int* cnt = nullptr;
      for (int l = 0; l < L; ++l)
        if ((s = dalloc(x, &wol[l], static_cast<size_t>(RT) * KTL * blk)) != NLD_OK) return s;
      const size_t zrows = 2ull * x->M_max;
      if ((s = dalloc(x, &attz, zrows * (x->qd + rpad) * el)) != NLD_OK) return s;
      const size_t ncnt = static_cast<size_t>((256 + 15) / 16) * ((x->M_max + 31) / 32);
      if ((s = dalloc(x, &cnt, ncnt * sizeof(int))) != NLD_OK) return s;
      CK(cudaMemsetAsync(attz, 0, zrows * (x->qd + rpad) * el, x->stream));
      CK(cudaMemsetAsync(cnt, 0, ncnt * sizeof(int), x->stream));
      x->wol.swap(wol);
      x->attz = attz;
      x->lora_cnt = cnt;
      x->lora_rpad = rpad;
      x->tmX.clear();
    }
    void* stage = nullptr;
    void* tiled = nullptr;
    CK(cudaMalloc(&stage, static_cast<size_t>(d) * rpad * el));
    if (cudaMalloc(&tiled, static_cast<size_t>(RT) * KB * blk) != cudaSuccess) {
      cudaFree(stage);
      return fail(x, NLD_ERR_CUDA, "out of device memory (adapter staging)");
    }
    cudaError_t e = cudaMemsetAsync(stage, 0, static_cast<size_t>(d) * rpad * el, x->stream);
    for (int l = 0; l < L && e == cudaSuccess; ++l) {
      e = cudaMemcpy2DAsync(x->wol[l], KTL * blk, x->wo[l], KT * blk, KT * blk, RT, cudaMemcpyDeviceToDevice,
                            x->stream);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(stage, rpad * el, x->lora_B[l], rank * el, rank * el, d, cudaMemcpyDeviceToDevice,
                              x->stream);
      if (e == cudaSuccess) e = launch_repack(x->stream, tiled, stage, nullptr, d, rpad, nullptr, true, true);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(static_cast<char*>(x->wol[l]) + KT * blk, KTL * blk, tiled, KB * blk, KB * blk, RT,
                              cudaMemcpyDeviceToDevice, x->stream);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(x->stream);
    cudaFree(stage);
    cudaFree(tiled);
    if (e != cudaSuccess) return fail(x, NLD_ERR_CUDA, "folding the adapter failed: %s", cudaGetErrorString(e));
  }
  CK(cudaStreamSynchronize(x->stream));
  x->lora_r = rank;
  x->lora_scale = scale;
  return NLD_OK;
}

nld_status nld_init_weights(nld_ctx* x, const void* const* tensors, int n_tensors, int on_device) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  const nld_config& c = x->c;
  const int L = c.n_layers;
  if (!tensors || n_tensors != 3 + 9 * L)
    return fail(x, NLD_ERR_ARG, "expected %d weight tensors, got %d", 3 + 9 * L, n_tensors);
  for (int i = 0; i < n_tensors; ++i)
    if (!tensors[i]) return fail(x, NLD_ERR_ARG, "weight tensor %d is NULL", i);
  const size_t el = x->el;
  const int d = c.d_model, F = c.ffn_dim, V = c.vocab, hd = c.head_dim;
  if (x->weights_ready) return fail(x, NLD_ERR_STATE, "weights already initialised");
  nld_status s;
  // allocations
  // bf16 matrices are stored pre-tiled (16 KB blocks), with rows padded to a multiple of 128
  auto pad = [&](int rows) { return x->bf16 ? (rows + kTileRows - 1) / kTileRows * kTileRows : rows; };
  const bool tiled = x->bf16;
  if ((s = dalloc(x, &x->embed, static_cast<size_t>(V + 1) * d * el)) != NLD_OK) return s;
  x->wqkv.resize(L);
  x->wo.resize(L);
  x->wgu.resize(L);
  x->wd.resize(L);
  for (int l = 0; l < L; ++l) {
    if ((s = dalloc(x, &x->wqkv[l], static_cast<size_t>(pad(x->qkv_rows)) * d * el)) != NLD_OK) return s;
    if ((s = dalloc(x, &x->wo[l], static_cast<size_t>(pad(d)) * x->qd * el)) != NLD_OK) return s;
    if ((s = dalloc(x, &x->wgu[l], static_cast<size_t>(pad(x->gu_rows)) * d * el)) != NLD_OK) return s;
    if ((s = dalloc(x, &x->wd[l], static_cast<size_t>(pad(d)) * F * el)) != NLD_OK) return s;
  }
  if ((s = dalloc(x, &x->wlm, static_cast<size_t>(pad(V)) * d * el)) != NLD_OK) return s;

  // row maps: q/k heads interleave (i, i+hd/2); gate/up interleave per 64 features
  std::vector<int> map_q(x->qd), map_kv(x->kvd), map_g(F), map_u(F);
  for (int r = 0; r < x->qd; ++r) {
    const int h = r / hd, lr = r % hd;
    map_q[r] = h * hd + ((lr & 1) ? (lr >> 1) + hd / 2 : (lr >> 1));
  }
  for (int r = 0; r < x->kvd; ++r) {
    const int h = r / hd, lr = r % hd;
    map_kv[r] = h * hd + ((lr & 1) ? (lr >> 1) + hd / 2 : (lr >> 1));
  }
  int *d_map_q = nullptr, *d_map_kv = nullptr, *d_map_gu = nullptr;
  std::vector<int> map_gu(2 * F);
  // destination row 128t + 2i <- gate 64t+i ; 128t + 2i + 1 <- up 64t+i (sources concatenated
  // as [Wg; Wu] in a staging buffer, so up rows are offset by F)
  for (int t = 0; t < F / 64; ++t)
    for (int i = 0; i < 64; ++i) {
      map_gu[128 * t + 2 * i] = 64 * t + i;
      map_gu[128 * t + 2 * i + 1] = F + 64 * t + i;
    }
  if ((s = dalloc(x, &d_map_q, x->qd * sizeof(int))) != NLD_OK) return s;
  if ((s = dalloc(x, &d_map_kv, x->kvd * sizeof(int))) != NLD_OK) return s;
  if ((s = dalloc(x, &d_map_gu, 2 * F * sizeof(int))) != NLD_OK) return s;
  CK(cudaMemcpy(d_map_q, map_q.data(), x->qd * sizeof(int), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(d_map_kv, map_kv.data(), x->kvd * sizeof(int), cudaMemcpyHostToDevice));
  CK(cudaMemcpy(d_map_gu, map_gu.data(), 2 * F * sizeof(int), cudaMemcpyHostToDevice));

  // staging: the largest source (embed/lm head or [Wg;Wu]) plus one gain vector
  size_t max_src = std::max({static_cast<size_t>(V + 1) * d, static_cast<size_t>(2) * F * d,
                             static_cast<size_t>(x->qd) * d, static_cast<size_t>(d) * F});
  void* stage = nullptr;
  void* stage_g = nullptr;
  if ((s = dalloc(x, &stage, max_src * el)) != NLD_OK) return s;
  if ((s = dalloc(x, &stage_g, static_cast<size_t>(d) * el)) != NLD_OK) return s;
  const cudaMemcpyKind kind = on_device ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  auto up = [&](const void* src, size_t n, void* dst) -> nld_status {
    CK(cudaMemcpyAsync(dst, src, n * el, kind, x->stream));
    return NLD_OK;
  };
  // embedding: plain copy
  TRY(up(tensors[0], static_cast<size_t>(V + 1) * d, x->embed));
  for (int l = 0; l < L; ++l) {
    const void* const* t = tensors + 1 + 9 * l;
    TRY(up(t[0], d, stage_g));
    char* qkv = static_cast<char*>(x->wqkv[l]);
    // q, k and v parts start on 128-row boundaries, where the tiled and row-major offsets agree
    TRY(up(t[1], static_cast<size_t>(x->qd) * d, stage));
    CK(launch_repack(x->stream, qkv, stage, d_map_q, x->qd, d, stage_g, x->bf16, tiled));
    TRY(up(t[2], static_cast<size_t>(x->kvd) * d, stage));
    CK(launch_repack(x->stream, qkv + static_cast<size_t>(x->qd) * d * el, stage, d_map_kv, x->kvd, d, stage_g, x->bf16, tiled));
    TRY(up(t[3], static_cast<size_t>(x->kvd) * d, stage));
    CK(launch_repack(x->stream, qkv + static_cast<size_t>(x->qd + x->kvd) * d * el, stage, nullptr, x->kvd, d, stage_g, x->bf16, tiled));
    TRY(up(t[4], static_cast<size_t>(d) * x->qd, stage));
    CK(launch_repack(x->stream, x->wo[l], stage, nullptr, d, x->qd, nullptr, x->bf16, tiled));
    TRY(up(t[5], d, stage_g));
    TRY(up(t[6], static_cast<size_t>(F) * d, stage));
    TRY(up(t[7], static_cast<size_t>(F) * d, static_cast<char*>(stage) + static_cast<size_t>(F) * d * el));
    CK(launch_repack(x->stream, x->wgu[l], stage, d_map_gu, 2 * F, d, stage_g, x->bf16, tiled));
    CK(cudaStreamSynchronize(x->stream));   // staging reuse
    TRY(up(t[8], static_cast<size_t>(d) * F, stage));
    CK(launch_repack(x->stream, x->wd[l], stage, nullptr, d, F, nullptr, x->bf16, tiled));
    CK(cudaStreamSynchronize(x->stream));
  }
  TRY(up(tensors[1 + 9 * L], d, stage_g));
  TRY(up(tensors[2 + 9 * L], static_cast<size_t>(V) * d, stage));
  CK(launch_repack(x->stream, x->wlm, stage, nullptr, V, d, stage_g, x->bf16, tiled));
  CK(cudaStreamSynchronize(x->stream));
  // release staging (the last allocations)
  for (void* p : {stage, stage_g, static_cast<void*>(d_map_q), static_cast<void*>(d_map_kv), static_cast<void*>(d_map_gu)}) {
    cudaFree(p);
    x->allocs.erase(std::remove(x->allocs.begin(), x->allocs.end(), p), x->allocs.end());
  }
  if (x->bf16) {
    x->tmWqkv.resize(L);
    x->tmWo.resize(L);
    x->tmWgu.resize(L);
    x->tmWd.resize(L);
    bool ok = true;
    for (int l = 0; l < L; ++l) {
      ok &= make_map_tiled(&x->tmWqkv[l], x->wqkv[l], x->qkv_rows, d);
      ok &= make_map_tiled(&x->tmWo[l], x->wo[l], d, x->qd);
      ok &= make_map_tiled(&x->tmWgu[l], x->wgu[l], x->gu_rows, d);
      ok &= make_map_tiled(&x->tmWd[l], x->wd[l], d, F);
    }
    ok &= make_map_tiled(&x->tmWlm, x->wlm, V, d);
    if (!ok) return fail(x, NLD_ERR_CUDA, "tensor map encode failed (weights)");
  }
  x->weights_ready = true;
  return NLD_OK;
}

namespace {
nld_status flush_fill(nld_ctx* x);   // (diffusion, below)
}  // namespace

nld_status nld_prefill(nld_ctx* x, const int32_t* d_tokens, int stride, const int32_t* d_lens, int batch,
                       int32_t* d_pending_out) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if (!x->weights_ready) return fail(x, NLD_ERR_STATE, "weights not initialised");
  if (!d_tokens) return fail(x, NLD_ERR_ARG, "tokens is NULL");
  if (batch < 1 || batch > x->c.max_batch) return fail(x, NLD_ERR_ARG, "batch %d outside 1..%d", batch, x->c.max_batch);
  if (stride < 1 || stride > x->c.max_seq) return fail(x, NLD_ERR_ARG, "prompt stride %d outside 1..%d", stride, x->c.max_seq);
  x->batch = batch;
  const int k = x->c.block_k;
  CK(cudaMemcpyAsync(x->prompt, d_tokens, static_cast<size_t>(batch) * stride * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  if (d_lens)
    CK(cudaMemcpyAsync(x->plens, d_lens, batch * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  else
    CK(launch_fill_i32(x->stream, x->plens, stride, batch));
  CK(cudaMemsetAsync(x->lens, 0, batch * sizeof(int), x->stream));
  CK(launch_fill_i32(x->stream, x->blk, x->c.vocab, batch * k));
  CK(launch_fill_i32(x->stream, x->draft, x->c.vocab, batch * k));
  CK(launch_fill_i32(x->stream, x->verify, -1, batch * (k + 1)));
  CK(cudaMemsetAsync(x->fillnext, 0, batch * sizeof(int), x->stream));
  x->nl_active = false;
  x->len_upper = 0;
  // causal forwards over positions 0..stride-2 in chunks of up to prefill_tokens rows; every
  // sequence advances by the chunk (rows past its own prompt are padding), and the last
  // finalize sets each sequence's length and pending token from its own prompt length
  const int chunk = std::max(1, x->prefill_tokens / batch);
  const int rows = stride - 1;
  int c0 = 0;
  do {
    const int m = std::min(chunk, rows - c0);
    const bool last = (c0 + m >= rows);
    if (m > 0) {
      FwdSpec f{};
      f.mode = FWD_PREFILL;
      f.B = batch;
      f.m = m;
      f.bs = 1;
      f.lm = LM_NONE;
      f.chunk0 = c0;
      f.prompt_len = stride;
      x->len_upper = c0;
      TRY(launch_forward(x, f));
    }
    FinalizeArgs a = base_fin(x, FWD_PREFILL, std::max(m, 1));
    a.chunk = m;
    a.prompt = last ? x->prompt : nullptr;
    a.prompt_len = stride;
    a.plens = x->plens;
    a.pending_out = last ? d_pending_out : nullptr;
    TRY(finalize(x, a));
    c0 += m;
    if (last) break;
  } while (true);
  x->len_upper = rows;
  x->started = true;
  x->verify_fresh = false;
  x->quad_ready = false;
  x->fill_pending = false;
  return NLD_OK;
}

nld_status nld_ar_step(nld_ctx* x, int32_t* d_tokens_out) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  TRY(ensure_capacity(x, 1));
  std::vector<uintptr_t> key = {1, static_cast<uintptr_t>(x->batch), reinterpret_cast<uintptr_t>(d_tokens_out)};
  const long long saved = x->len_upper;
  TRY(run_graph(x, key, [&]() -> nld_status {
    FwdSpec f{};
    f.mode = FWD_AR;
    f.B = x->batch;
    f.m = 1;
    f.bs = 1;
    f.lm = LM_ARGMAX;
    x->len_upper = x->c.max_seq;   // graphs are sized for the longest sequence
    nld_status s = launch_forward(x, f);
    x->len_upper = saved;
    if (s != NLD_OK) return s;
    FinalizeArgs a = base_fin(x, FWD_AR, 1);
    a.tokens_out = d_tokens_out;
    return finalize(x, a);
  }));
  x->len_upper += 1;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

static nld_status draft_verify_body(nld_ctx* x) {
  const int k = x->c.block_k;
  const long long saved = x->len_upper;
  x->len_upper = x->c.max_seq;
  FwdSpec f{};
  f.mode = FWD_DRAFT;
  f.B = x->batch;
  f.m = k;
  f.bs = k;
  f.lm = LM_ARGMAX;
  nld_status s = launch_forward(x, f);
  if (s == NLD_OK) s = finalize(x, base_fin(x, FWD_DRAFT, k));
  if (s == NLD_OK) {
    f.mode = FWD_VERIFY;
    f.m = k + 1;
    f.bs = 1;
    s = launch_forward(x, f);
  }
  if (s == NLD_OK) s = finalize(x, base_fin(x, FWD_VERIFY, k + 1));
  x->len_upper = saved;
  return s;
}

nld_status nld_selfspec_draft_verify(nld_ctx* x) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  TRY(ensure_capacity(x, x->c.block_k + 1));
  std::vector<uintptr_t> key = {2, static_cast<uintptr_t>(x->batch)};
  TRY(run_graph(x, key, [&]() { return draft_verify_body(x); }));
  x->verify_fresh = true;
  x->quad_ready = false;
  return NLD_OK;
}

nld_status nld_kv_commit(nld_ctx* x, const int32_t* d_nrows, int32_t* d_tokens_out, int32_t* d_ncommit_out) {
  TRY(need_started(x));
  if (!x->verify_fresh) return fail(x, NLD_ERR_STATE, "no uncommitted verify forward");
  FinalizeArgs a = base_fin(x, FWD_COMMIT, x->c.block_k + 1);
  a.force = d_nrows;
  a.tokens_out = d_tokens_out;
  a.ncommit_out = d_ncommit_out;
  TRY(finalize(x, a));
  x->len_upper += x->c.block_k + 1;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

nld_status nld_selfspec_round(nld_ctx* x, int32_t* d_tokens_out, int32_t* d_ncommit_out,
                              const int32_t* d_force_ncommit) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  TRY(ensure_capacity(x, x->c.block_k + 1));
  std::vector<uintptr_t> key = {3, static_cast<uintptr_t>(x->batch), reinterpret_cast<uintptr_t>(d_tokens_out),
                                reinterpret_cast<uintptr_t>(d_ncommit_out), reinterpret_cast<uintptr_t>(d_force_ncommit)};
  TRY(run_graph(x, key, [&]() -> nld_status {
    TRY(draft_verify_body(x));
    FinalizeArgs a = base_fin(x, FWD_COMMIT, x->c.block_k + 1);
    a.force = d_force_ncommit;
    a.tokens_out = d_tokens_out;
    a.ncommit_out = d_ncommit_out;
    return finalize(x, a);
  }));
  x->len_upper += x->c.block_k + 1;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

// The quadratic self-speculation forward over the current drafts (no finalize): (k+1)^2 rows per
// sequence, the verify rows and the k+1 pre-draft blocks.
static nld_status quad_forward(nld_ctx* x, int lm, float* logits) {
  const int k = x->c.block_k;
  FwdSpec f{};
  f.mode = FWD_QUAD;
  f.B = x->batch;
  f.m = (k + 1) * (k + 1);
  f.bs = 1;
  f.causal_rows = k + 1;   // the verify rows; the LoRA drafter takes the pre-draft rows
  f.quad_k = k;
  f.lm = lm;
  f.logits = logits;
  return launch_forward(x, f);
}

// Checks shared by the quadratic entry points: the forward's batch x (k+1)^2 rows fit the
// activation buffers, and its rows' K/V slots (len .. len+(k+1)^2-1) fit the KV capacity.
static nld_status quad_check(nld_ctx* x) {
  const int k = x->c.block_k, m = (k + 1) * (k + 1);
  if (static_cast<long long>(x->batch) * m > x->M_max)
    return fail(x, NLD_ERR_UNSUPPORTED, "a quadratic forward needs batch x (k+1)^2 = %d x %d rows <= %d",
                x->batch, m, x->M_max);
  return ensure_capacity(x, m - k - 1);   // kv_cap >= max_seq + k + 1
}

nld_status nld_quadratic_round(nld_ctx* x, int32_t* d_tokens_out, int32_t* d_ncommit_out) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  TRY(quad_check(x));
  const int k = x->c.block_k;
  if (!x->quad_ready) {
    // the first round after any other call starts from one linear draft forward
    std::vector<uintptr_t> dkey = {11, static_cast<uintptr_t>(x->batch)};
    TRY(run_graph(x, dkey, [&]() -> nld_status {
      const long long saved = x->len_upper;
      x->len_upper = x->c.max_seq;
      FwdSpec f{};
      f.mode = FWD_DRAFT;
      f.B = x->batch;
      f.m = k;
      f.bs = k;
      f.lm = LM_ARGMAX;
      nld_status s = launch_forward(x, f);
      x->len_upper = saved;
      if (s != NLD_OK) return s;
      return finalize(x, base_fin(x, FWD_DRAFT, k));
    }));
  }
  std::vector<uintptr_t> key = {10, static_cast<uintptr_t>(x->batch), reinterpret_cast<uintptr_t>(d_tokens_out),
                                reinterpret_cast<uintptr_t>(d_ncommit_out)};
  TRY(run_graph(x, key, [&]() -> nld_status {
    const long long saved = x->len_upper;
    x->len_upper = x->c.max_seq;
    nld_status s = quad_forward(x, LM_ARGMAX, nullptr);
    x->len_upper = saved;
    if (s != NLD_OK) return s;
    FinalizeArgs a = base_fin(x, FWD_QUAD, (k + 1) * (k + 1));
    a.tokens_out = d_tokens_out;
    a.ncommit_out = d_ncommit_out;
    return finalize(x, a);
  }));
  x->len_upper += k + 1;
  x->verify_fresh = false;
  x->quad_ready = true;
  return NLD_OK;
}

namespace {

// The causal KV-fill forward of a complete diffusion block: len += k, pending = b_k.
nld_status run_fill(nld_ctx* x) {
  const int k = x->c.block_k;
  TRY(ensure_capacity(x, k));
  std::vector<uintptr_t> fkey = {5, static_cast<uintptr_t>(x->batch)};
  TRY(run_graph(x, fkey, [&]() -> nld_status {
    const long long saved = x->len_upper;
    x->len_upper = x->c.max_seq;
    FwdSpec f{};
    f.mode = FWD_FILL;
    f.B = x->batch;
    f.m = k;
    f.bs = 1;
    f.lm = LM_NONE;
    nld_status s = launch_forward(x, f);
    x->len_upper = saved;
    if (s != NLD_OK) return s;
    return finalize(x, base_fin(x, FWD_FILL, k));
  }));
  x->len_upper += k;
  x->fill_pending = false;
  return NLD_OK;
}

// One forward of per-sequence diffusion: sequences flagged in fillnext run their causal KV
// fill, the others denoise (fill_only: keep their state, no LM head).
nld_status run_nl(nld_ctx* x, bool fill_only, float threshold, int32_t* d_block_out, float* d_conf_out,
                  int32_t* d_ncommit_out, int32_t* d_state_out) {
  const int k = x->c.block_k;
  TRY(ensure_capacity(x, k));
  uint32_t thr_bits;
  std::memcpy(&thr_bits, &threshold, 4);
  std::vector<uintptr_t> key = {static_cast<uintptr_t>(fill_only ? 9 : 8), static_cast<uintptr_t>(x->batch),
                                reinterpret_cast<uintptr_t>(d_block_out), reinterpret_cast<uintptr_t>(d_conf_out),
                                reinterpret_cast<uintptr_t>(d_ncommit_out), reinterpret_cast<uintptr_t>(d_state_out),
                                thr_bits};
  TRY(run_graph(x, key, [&]() -> nld_status {
    const long long saved = x->len_upper;
    x->len_upper = x->c.max_seq;
    FwdSpec f{};
    f.mode = fill_only ? FWD_NLFILL : FWD_NLDIFF;
    f.B = x->batch;
    f.m = k;
    f.bs = k;
    f.causal_seq = x->fillnext;
    f.lm = fill_only ? LM_NONE : LM_ARGMAX;
    nld_status s = launch_forward(x, f);
    x->len_upper = saved;
    if (s != NLD_OK) return s;
    FinalizeArgs a = base_fin(x, f.mode, k);
    a.threshold = threshold;
    a.block_out = d_block_out;
    a.conf_out = d_conf_out;
    a.ncommit_out = d_ncommit_out;
    a.state_out = d_state_out;
    a.incomplete = nullptr;
    return finalize(x, a);
  }));
  x->len_upper += k;   // upper bound: a fill grows a sequence by k
  return NLD_OK;
}

// Fills that per-sequence diffusion left due run before any other decode call: one forward,
// only if some sequence is flagged.
nld_status flush_nl(nld_ctx* x) {
  if (!x->nl_active) return NLD_OK;
  int* flags = x->h_pinned + 2 + x->batch;
  CK(cudaMemcpyAsync(flags, x->fillnext, sizeof(int) * x->batch, cudaMemcpyDeviceToHost, x->stream));
  CK(cudaStreamSynchronize(x->stream));
  bool any = false;
  for (int b = 0; b < x->batch; ++b) any = any || flags[b] != 0;
  if (any) TRY(run_nl(x, true, 0.f, nullptr, nullptr, nullptr, nullptr));
  x->nl_active = false;   // only once the due fills ran: a failed flush is retried next call
  return NLD_OK;
}

// A deferred fill (lockstep or per-sequence) runs alone before any other decode call.
nld_status flush_fill(nld_ctx* x) {
  TRY(flush_nl(x));
  return x->fill_pending ? run_fill(x) : NLD_OK;
}

// One denoising forward + commit (fused = the deferred fill of the previous block and the new
// block's first step in one forward of 2k rows); returns the number of sequences whose block
// is still open.
nld_status run_denoise(nld_ctx* x, bool fused, float threshold, int32_t* d_block_out, float* d_conf_out,
                       int32_t* d_ncommit_out, int* open_out) {
  const int k = x->c.block_k;
  uint32_t thr_bits;
  std::memcpy(&thr_bits, &threshold, 4);
  std::vector<uintptr_t> key = {static_cast<uintptr_t>(fused ? 6 : 4), static_cast<uintptr_t>(x->batch),
                                reinterpret_cast<uintptr_t>(d_block_out), reinterpret_cast<uintptr_t>(d_conf_out),
                                reinterpret_cast<uintptr_t>(d_ncommit_out), thr_bits};
  TRY(run_graph(x, key, [&]() -> nld_status {
    CK(cudaMemsetAsync(x->incomplete, 0, sizeof(int), x->stream));
    const long long saved = x->len_upper;
    x->len_upper = x->c.max_seq;
    FwdSpec f{};
    f.mode = fused ? FWD_FILLDIFF : FWD_DIFFUSE;
    f.B = x->batch;
    f.m = fused ? 2 * k : k;
    f.bs = k;
    f.causal_rows = fused ? k : 0;
    f.lm = LM_ARGMAX;
    nld_status s = launch_forward(x, f);
    x->len_upper = saved;
    if (s != NLD_OK) return s;
    FinalizeArgs a = base_fin(x, f.mode, f.m);
    a.threshold = threshold;
    a.block_out = d_block_out;
    a.conf_out = d_conf_out;
    a.ncommit_out = d_ncommit_out;
    TRY(finalize(x, a));
    CK(cudaMemcpyAsync(x->h_pinned + 1, x->incomplete, sizeof(int), cudaMemcpyDeviceToHost, x->stream));
    return NLD_OK;
  }));
  CK(cudaStreamSynchronize(x->stream));
  *open_out = x->h_pinned[1];
  return NLD_OK;
}

}  // namespace

nld_status nld_diffuse_block_step(nld_ctx* x, float threshold, int32_t* d_block_out, float* d_conf_out,
                                  int32_t* d_ncommit_out, int32_t* h_filled_out) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  TRY(ensure_capacity(x, x->c.block_k));
  int open = 1;
  TRY(run_denoise(x, false, threshold, d_block_out, d_conf_out, d_ncommit_out, &open));
  int filled = 0;
  if (open == 0) {
    TRY(run_fill(x));
    filled = 1;
  }
  if (h_filled_out) *h_filled_out = filled;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

// Largest forward (batch x 2k token rows) that runs the fused fill as one forward.
constexpr int kFusedFillRows = 256;

nld_status nld_diffuse_block_step_fused(nld_ctx* x, float threshold, int32_t* d_block_out,
                                        float* d_conf_out, int32_t* d_ncommit_out, int32_t* h_filled_out) {
  TRY(need_started(x));
  TRY(flush_nl(x));
  const int k = x->c.block_k;
  const bool filling = x->fill_pending;
  if (filling && (2 * k > 64 || x->batch * 2 * k > x->M_max))
    return fail(x, NLD_ERR_UNSUPPORTED, "fused fill needs 2k <= 64 and batch*2k <= %d rows", x->M_max);
  // The 2k-row forward saves a weight stream while the forward is bound by HBM; past
  // kFusedFillRows token rows the (hi, lo) products make it compute-bound and it costs as much
  // as the two forwards it replaces, so the fill then runs alone first (same results: the two
  // forms are equal in exact arithmetic)
  const bool fused = filling && x->batch * 2 * k <= kFusedFillRows;
  if (filling && !fused) TRY(run_fill(x));
  TRY(ensure_capacity(x, fused ? 2 * k : k));
  int open = 1;
  TRY(run_denoise(x, fused, threshold, d_block_out, d_conf_out, d_ncommit_out, &open));
  if (fused) {
    x->len_upper += k;
    x->fill_pending = false;
  }
  if (open == 0) x->fill_pending = true;   // this block's fill joins the next step
  if (h_filled_out) *h_filled_out = filling ? 1 : 0;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

nld_status nld_diffuse_step_nonlockstep(nld_ctx* x, float threshold, int32_t* d_block_out, float* d_conf_out,
                                        int32_t* d_ncommit_out, int32_t* d_state_out) {
  TRY(need_started(x));
  if (x->fill_pending) TRY(run_fill(x));   // a lockstep block's deferred fill
  TRY(run_nl(x, false, threshold, d_block_out, d_conf_out, d_ncommit_out, d_state_out));
  x->nl_active = true;
  x->verify_fresh = false;
  x->quad_ready = false;
  return NLD_OK;
}

nld_status nld_debug_logits(nld_ctx* x, int mode, float* d_logits_out) {
  TRY(need_started(x));
  TRY(flush_fill(x));
  if (!d_logits_out) return fail(x, NLD_ERR_ARG, "logits is NULL");
  const int k = x->c.block_k;
  if (mode == NLD_MODE_QUAD) {
    // the quadratic forward over the current drafts; nothing is recorded or committed
    TRY(quad_check(x));
    TRY(quad_forward(x, LM_LOGITS, d_logits_out));
    x->quad_ready = false;
    return NLD_OK;
  }
  FwdSpec f{};
  f.B = x->batch;
  f.lm = LM_LOGITS;
  f.logits = d_logits_out;
  int fm;
  switch (mode) {
    case NLD_MODE_AR: fm = FWD_AR; f.m = 1; f.bs = 1; break;
    case NLD_MODE_DRAFT: fm = FWD_DRAFT; f.m = k; f.bs = k; break;
    case NLD_MODE_VERIFY: fm = FWD_VERIFY; f.m = k + 1; f.bs = 1; break;
    case NLD_MODE_DIFFUSE: fm = FWD_DIFFUSE; f.m = k; f.bs = k; break;
    default: return fail(x, NLD_ERR_ARG, "unknown mode %d", mode);
  }
  TRY(ensure_capacity(x, f.m));
  f.mode = fm;
  TRY(launch_forward(x, f));
  // also record argmaxes (drafts / verify) through the argmax epilogue of the same forward
  f.lm = LM_ARGMAX;
  f.logits = nullptr;
  TRY(launch_forward(x, f));
  FinalizeArgs a = base_fin(x, fm, f.m);
  a.commit = 0;
  TRY(finalize(x, a));
  x->quad_ready = false;
  if (mode == NLD_MODE_VERIFY) x->verify_fresh = true;
  return NLD_OK;
}

static ProjRef hook_proj(nld_ctx* x, int which, int layer, int M) {
  const int m = M / x->batch;
  ProjRef r{which, layer, base_epi(x, M, m)};
  static const int kinds[5] = {EPI_QKV, EPI_RESID, EPI_SWIGLU, EPI_RESID, EPI_LMHEAD};
  r.e.kind = kinds[which];
  r.e.kv_layer = static_cast<char*>(x->pool) + static_cast<size_t>(layer) * x->layer_elems * x->el;
  return r;
}

nld_status nld_time_gemm(nld_ctx* x, int which, int layer, int M, int reps, float* ms_out) {
  TRY(need_started(x));
  if (which < 0 || which > 4) return fail(x, NLD_ERR_ARG, "which must be 0..4");
  if (layer < 0 || layer >= x->c.n_layers) return fail(x, NLD_ERR_ARG, "layer out of range");
  if (M < 1 || M > x->M_max || M % x->batch) return fail(x, NLD_ERR_ARG, "M must be a multiple of the batch, <= %d", x->M_max);
  if (reps < 1 || !ms_out) return fail(x, NLD_ERR_ARG, "reps >= 1 and ms_out required");
  TRY(ensure_capacity(x, M / x->batch));
  const ProjRef r = hook_proj(x, which, layer, M);
  cudaEvent_t a, b;
  CK(cudaEventCreate(&a));
  CK(cudaEventCreate(&b));
  TRY(chain(x, &r, 1, M, false, x->bars, nullptr, 0));   // warm (tensor maps, first-launch costs)
  CK(cudaEventRecord(a, x->stream));
  for (int i = 0; i < reps; ++i) TRY(chain(x, &r, 1, M, false, x->bars, nullptr, 0));
  CK(cudaEventRecord(b, x->stream));
  CK(cudaEventSynchronize(b));
  float ms = 0.f;
  CK(cudaEventElapsedTime(&ms, a, b));
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  *ms_out = ms / reps;
  return NLD_OK;
}

nld_status nld_trace_gemm(nld_ctx* x, int which, int layer, int M, unsigned long long* d_trace,
                          int* grid_out) {
  TRY(need_started(x));
  if (!x->bf16) return fail(x, NLD_ERR_UNSUPPORTED, "tensor-core GEMM only");
  if (which < 0 || which > 4 || layer < 0 || layer >= x->c.n_layers || !d_trace || M < 1 ||
      M > x->M_max || M % x->batch)
    return fail(x, NLD_ERR_ARG, "bad trace arguments");
  const ProjRef r = hook_proj(x, which, layer, M);
  int grid = 0;
  plan_chain(x, &r, 1, M, &grid);
  if (grid_out) *grid_out = grid;
  TRY(chain(x, &r, 1, M, false, x->bars, nullptr, 0));
  TRY(chain(x, &r, 1, M, false, x->bars, nullptr, 0, d_trace));
  CK(cudaStreamSynchronize(x->stream));
  return NLD_OK;
}

nld_status nld_trace_chain(nld_ctx* x, int layer, int M, unsigned long long* d_trace, int* grid_out) {
  TRY(need_started(x));
  if (!x->bf16) return fail(x, NLD_ERR_UNSUPPORTED, "tensor-core GEMM only");
  if (layer < 0 || layer + 1 >= x->c.n_layers || !d_trace || M < 1 || M > x->M_max || M % x->batch)
    return fail(x, NLD_ERR_ARG, "bad trace arguments");
  TRY(ensure_capacity(x, M / x->batch));
  ProjRef pr[4] = {hook_proj(x, GW_O, layer, M), hook_proj(x, GW_GU, layer, M),
                   hook_proj(x, GW_D, layer, M), hook_proj(x, GW_QKV, layer + 1, M)};
  int grid = 0;
  plan_chain(x, pr, 4, M, &grid);
  if (grid_out) *grid_out = grid;
  unsigned* bar = x->bars + (1 + layer) * kMaxPhases;
  TRY(chain(x, pr, 4, M, false, bar, nullptr, 0));
  TRY(chain(x, pr, 4, M, false, bar, nullptr, 0, d_trace));
  CK(cudaStreamSynchronize(x->stream));
  return NLD_OK;
}

nld_status nld_time_chain(nld_ctx* x, int layer, int M, int reps, float* ms_out) {
  TRY(need_started(x));
  if (!x->bf16) return fail(x, NLD_ERR_UNSUPPORTED, "tensor-core GEMM only");
  if (layer < 0 || layer + 1 >= x->c.n_layers || M < 1 || M > x->M_max || M % x->batch || reps < 1 || !ms_out)
    return fail(x, NLD_ERR_ARG, "bad timing arguments");
  TRY(ensure_capacity(x, M / x->batch));
  ProjRef pr[4] = {hook_proj(x, GW_O, layer, M), hook_proj(x, GW_GU, layer, M),
                   hook_proj(x, GW_D, layer, M), hook_proj(x, GW_QKV, layer + 1, M)};
  unsigned* bar = x->bars + (1 + layer) * kMaxPhases;
  cudaEvent_t a, b;
  CK(cudaEventCreate(&a));
  CK(cudaEventCreate(&b));
  TRY(chain(x, pr, 4, M, false, bar, nullptr, 0));
  CK(cudaEventRecord(a, x->stream));
  for (int i = 0; i < reps; ++i) TRY(chain(x, pr, 4, M, false, bar, nullptr, 0));
  CK(cudaEventRecord(b, x->stream));
  CK(cudaEventSynchronize(b));
  float ms = 0.f;
  CK(cudaEventElapsedTime(&ms, a, b));
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  *ms_out = ms / reps;
  return NLD_OK;
}

nld_status nld_debug_chain_tuning(nld_ctx* x, int stage_cap, int k_tiles_per_stage, int boundary_prefetch,
                                  int act_3d, int runahead_stages, int warm_next) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if (stage_cap < 0 || stage_cap == 1 || stage_cap == 2 || stage_cap > gemm_chain_max_stages() ||
      k_tiles_per_stage < 0 || k_tiles_per_stage > 2 || boundary_prefetch < 0 || boundary_prefetch > 256 ||
      (act_3d != 0 && act_3d != 1) || runahead_stages < 0 || runahead_stages > 16 || warm_next < 0 ||
      warm_next > 256)
    return fail(x, NLD_ERR_ARG,
                "stage cap 0 or 3..%d, k-tiles per stage 0..2, boundary prefetch 0..256, act_3d 0/1, "
                "run-ahead 0..16, warm-next 0..256",
                gemm_chain_max_stages());
  CK(cudaStreamSynchronize(x->stream));
  drop_graphs(x);   // captured graphs hold the old launch parameters
  x->chain_stage_cap = stage_cap;
  x->chain_kps = k_tiles_per_stage;
  x->chain_boundary_pf = boundary_prefetch;
  if (x->chain_x3d != act_3d) x->tmX.clear();   // activation maps of the other form
  x->chain_x3d = act_3d;
  x->chain_pf_stages = runahead_stages;
  x->chain_warm_next = warm_next;
  return NLD_OK;
}

nld_status nld_debug_layer_trace(nld_ctx* x, int layer, unsigned long long* d_attn_trace, size_t n_attn,
                                 unsigned long long* d_chain_trace, size_t n_chain) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if (layer >= x->c.n_layers || (d_attn_trace == nullptr) != (n_attn == 0) ||
      (d_chain_trace != nullptr && n_chain < kChainTraceEntries))
    return fail(x, NLD_ERR_ARG, "layer < n_layers; attention buffer and size both or neither; chain buffer >= %d entries",
                kChainTraceEntries);
  CK(cudaStreamSynchronize(x->stream));
  drop_graphs(x);   // captured graphs hold the old launch parameters
  x->trace_layer = layer < 0 ? -1 : layer;
  x->attn_trace = layer < 0 ? nullptr : d_attn_trace;
  x->attn_trace_n = layer < 0 ? 0 : n_attn;
  x->chain_trace = layer < 0 ? nullptr : d_chain_trace;
  return NLD_OK;
}

nld_status nld_debug_attention_kernel(int kernel) {
  if (kernel < 0 || kernel > 4)
    return fail(nullptr, NLD_ERR_ARG, "0 (planner), 1 (tcgen05), 2 (mma.sync), 3 / 4 (tcgen05, 2 / 4 threads per row)");
  g_attn_kernel.store(kernel);
  return NLD_OK;
}

nld_status nld_debug_attention_tile(int keys) {
  if (keys != 0 && keys != 64 && keys != 128)
    return fail(nullptr, NLD_ERR_ARG, "keys per tcgen05 KV tile: 0 (planner), 64 or 128");
  g_attn_tile.store(keys);
  return NLD_OK;
}

nld_status nld_debug_attention_tuning(nld_ctx* x, int rows_per_cta, int min_tiles_per_split) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  if ((rows_per_cta != 0 && (rows_per_cta < 16 || rows_per_cta > 144)) || min_tiles_per_split < 0 ||
      min_tiles_per_split > 8)
    return fail(x, NLD_ERR_ARG, "rows per CTA 0 or 16..144, KV tiles per split 0..8");
  CK(cudaStreamSynchronize(x->stream));
  drop_graphs(x);
  x->attn_rows_cap = rows_per_cta;
  x->attn_min_tiles = min_tiles_per_split;
  return NLD_OK;
}

nld_status nld_debug_timeout_chain(nld_ctx* x, unsigned long long timeout_ns) {
  TRY(need_started(x));
  if (!x->bf16) return fail(x, NLD_ERR_UNSUPPORTED, "tensor-core GEMM only");
  if (x->c.n_layers < 2) return fail(x, NLD_ERR_UNSUPPORTED, "needs two layers (a four-phase chain)");
  if (timeout_ns < 1000 || timeout_ns > 2000000000ull) return fail(x, NLD_ERR_ARG, "timeout outside 1 us..2 s");
  const int M = x->batch;
  TRY(ensure_capacity(x, 1));
  ProjRef pr[4] = {hook_proj(x, GW_O, 0, M), hook_proj(x, GW_GU, 0, M), hook_proj(x, GW_D, 0, M),
                   hook_proj(x, GW_QKV, 1, M)};
  int grid = 0;
  ChainArgs A = plan_chain(x, pr, 4, M, &grid);
  for (int p = 0; p < 4; ++p) {
    const WInfo w = winfo(x, pr[p].which, pr[p].layer);
    A.ph[p].tmW = *w.map;
    A.ph[p].W = w.W;
    int is3d = 0;
    const CUtensorMap* tmX = xmap(x, w.buf, A.xr, A.kps, &is3d);
    if (!tmX) return fail(x, NLD_ERR_CUDA, "tensor map encode failed (activation buffer)");
    A.ph[p].tmX = *tmX;
    A.ph[p].x3d = is3d;
    A.ph[p].e = pr[p].e;
    A.ph[p].e.n_rows = w.n_rows;
  }
  A.bar = x->bars + kMaxPhases;   // layer 0's counters (left zero by every launch)
  A.boundary_pf = x->chain_boundary_pf;
  A.pf_stages = x->chain_pf_stages;
  A.dbg_skip_arrive = 1;
  CK(launch_gemm_chain(x->stream, A, grid, timeout_ns, false));
  return NLD_OK;
}

nld_status nld_plan_chain(int M, int nph, const int* n_rows, const int* K, const int* max_clusters,
                          int hilo, int* out20) {
  if (!n_rows || !K || !max_clusters || !out20) return fail(nullptr, NLD_ERR_ARG, "NULL argument");
  if (M < 1 || nph < 1 || nph > kMaxPhases) return fail(nullptr, NLD_ERR_ARG, "bad plan sizes");
  for (int p = 0; p < nph; ++p)
    if (n_rows[p] < 1 || K[p] < kTileK || K[p] % kTileK)
      return fail(nullptr, NLD_ERR_ARG, "phase %d: rows %d, K %d", p, n_rows[p], K[p]);
  int grid = 0;
  const ChainArgs A = plan_chain_shapes(max_clusters, n_rows, K, nph, M, hilo ? 1 : 0, &grid);
  if (A.CS < 1) return fail(nullptr, NLD_ERR_UNSUPPORTED, "no cluster size can be resident");
  for (int i = 0; i < 20; ++i) out20[i] = 0;
  out20[0] = A.CS;
  out20[1] = A.NT;
  out20[2] = A.xr;
  out20[3] = A.kps;
  out20[4] = A.stages;
  out20[5] = A.slots;
  out20[6] = static_cast<int>(A.tmem_cols);
  out20[7] = grid;
  out20[8] = static_cast<int>(gemm_chain_smem_bytes(A.NT, A.NT << A.hilo, A.xr, A.kps, A.stages, A.CS, A.slots));
  out20[9] = A.ph[0].tok_tiles;
  for (int p = 0; p < nph; ++p) {
    out20[10 + 2 * p] = A.ph[p].s;
    out20[11 + 2 * p] = A.ph[p].ks;
  }
  return NLD_OK;
}

nld_status nld_plan_attention(int batch, int m, int Hq, int Hkv, int max_len, int sms, int* out8) {
  if (!out8) return fail(nullptr, NLD_ERR_ARG, "NULL argument");
  if (batch < 1 || m < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || max_len < 1 || sms < 1)
    return fail(nullptr, NLD_ERR_ARG, "bad attention plan sizes");
  AttnArgs a{};
  // pure host: clusters of S resident at once as if every SM held as many CTAs as its 228 KB of
  // shared memory allows (one block reserves 1 KB)
  attn_plan(batch, m, Hq, Hkv, max_len, sms, a, [sms](int S, int NW, int stages, int tc) {
    const size_t smem = tc ? attn_tc_smem_bytes(true, tc) : attn_mma_smem_bytes(NW, true, stages);
    const int per_sm = static_cast<int>(233472 / (smem + 1024));
    return std::max(1, sms * per_sm / S);
  }, 0, 0, g_attn_kernel.load(), g_attn_tile.load());
  const int v[8] = {a.G, a.QT, a.q_tiles, a.rows, a.NW, a.S, a.tc ? 1 : 0, a.tc ? a.tc_tile : 64};
  for (int i = 0; i < 8; ++i) out8[i] = v[i];
  return NLD_OK;
}

nld_status nld_debug_gemm_plan(nld_ctx* x, int which, int M, int* out8) {
  if (!x || !out8) return fail(x, NLD_ERR_ARG, "NULL argument");
  if (!x->bf16) return fail(x, NLD_ERR_UNSUPPORTED, "tensor-core GEMM only");
  if (which < 0 || which > 4 || M < 1 || M > x->M_max) return fail(x, NLD_ERR_ARG, "bad plan arguments");
  const ProjRef r{which, 0, base_epi(x, M, 1)};
  int grid = 0;
  const ChainArgs A = plan_chain(x, &r, 1, M, &grid);
  const int v[8] = {A.NT, A.ph[0].tok_tiles, A.ph[0].row_tiles, A.ph[0].KT, A.ph[0].s, A.ph[0].ks, grid, A.stages};
  for (int i = 0; i < 8; ++i) out8[i] = v[i];
  return NLD_OK;
}

nld_status nld_debug_state(nld_ctx* x, int32_t* d_lens_out, int32_t* d_pending_out, int32_t* d_draft_out,
                           int32_t* d_verify_out) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  const int B = std::max(x->batch, 1), k = x->c.block_k;
  if (d_lens_out) CK(cudaMemcpyAsync(d_lens_out, x->lens, B * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  if (d_pending_out) CK(cudaMemcpyAsync(d_pending_out, x->pending, B * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  if (d_draft_out) CK(cudaMemcpyAsync(d_draft_out, x->draft, static_cast<size_t>(B) * k * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  if (d_verify_out) CK(cudaMemcpyAsync(d_verify_out, x->verify, static_cast<size_t>(B) * (k + 1) * sizeof(int), cudaMemcpyDeviceToDevice, x->stream));
  return NLD_OK;
}

nld_status nld_sync(nld_ctx* x) {
  if (!x) return fail(nullptr, NLD_ERR_ARG, "ctx is NULL");
  CK(cudaMemcpyAsync(x->h_pinned, x->err, sizeof(int), cudaMemcpyDeviceToHost, x->stream));
  CK(cudaMemsetAsync(x->err, 0, sizeof(int), x->stream));
  CK(cudaStreamSynchronize(x->stream));
  const int e = x->h_pinned[0];
  if (e & NLD_DEVERR_TIMEOUT) return fail(x, NLD_ERR_TIMEOUT, "a bounded device wait ran out (error word 0x%x)", e);
  if (e & NLD_DEVERR_KV_OVERFLOW) return fail(x, NLD_ERR_KV_FULL, "a KV write past capacity was skipped (error word 0x%x)", e);
  if (e) return fail(x, NLD_ERR_DEVICE, "device bounds check failed (error word 0x%x)", e);
  return NLD_OK;
}

const char* nld_last_error(const nld_ctx* x) {
  return x ? x->msg.c_str() : g_static_err.c_str();
}

void* nld_stream(nld_ctx* x) { return x ? static_cast<void*>(x->stream) : nullptr; }

// -------------------------------------------------------------- stand-alone LM head (a8) --
// Resident clusters per split size on the current device (one GEMM CTA per SM), cached.
static const int* device_max_clusters() {
  static int cache[64][9];
  static bool ready[64] = {false};
  static std::mutex mu;   // callers may come from several threads
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    dev = 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!ready[dev]) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaGetLastError();
    cache[dev][0] = 0;
    for (int sp = 1; sp <= 8; ++sp) cache[dev][sp] = gemm_tc_max_clusters(sp, 200 * 1024, sms);
    ready[dev] = true;
  }
  return cache[dev];
}

// Workspace layout of the stand-alone LM head: a 256-byte block holding the device error word
// (bounded waits that ran out), then the per-tile RMS sums, then the per-(row, vocab tile) partials.
constexpr size_t kLmErrBytes = 256;
static size_t lm_ssq_bytes(int M, int d) { return (static_cast<size_t>(d / kTileRows) * M * sizeof(float) + 255) / 256 * 256; }
static size_t lm_part_bytes(int M, int vocab) {
  return static_cast<size_t>(M) * ((vocab + kTileRows - 1) / kTileRows) * sizeof(LmPart);
}

static nld_status lm_head_check(const void* h, const void* w, int M, int d, int vocab, const int32_t* am,
                                const float* cf) {
  if (!h || !w || !am || !cf) return fail(nullptr, NLD_ERR_ARG, "NULL pointer argument");
  if (M < 1 || M > 4096) return fail(nullptr, NLD_ERR_ARG, "M must be in 1..4096");
  if (d < 128 || d % 128) return fail(nullptr, NLD_ERR_ARG, "d must be a positive multiple of 128");
  if (vocab < 1) return fail(nullptr, NLD_ERR_ARG, "vocab must be >= 1");
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w)) % 16)
    return fail(nullptr, NLD_ERR_ARG, "hidden and weight must be 16-byte aligned");
  return NLD_OK;
}

// Launch the a8 path over caller buffers with scratch at ws (ssq then LM-head partials).
static nld_status lm_head_launch(const void* d_hidden, const void* d_lm_weight, int M, int d, int vocab,
                                 float rms_eps, int32_t* d_argmax_out, float* d_conf_out, char* ws,
                                 cudaStream_t st) {
  cudaError_t ae = init_kernel_attributes();
  if (ae != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, NLD_ERR_CUDA, "setting kernel shared-memory limits failed: %s", cudaGetErrorString(ae));
  }
  int* err = reinterpret_cast<int*>(ws);
  float* ssq = reinterpret_cast<float*>(ws + kLmErrBytes);
  LmPart* part = reinterpret_cast<LmPart*>(ws + kLmErrBytes + lm_ssq_bytes(M, d));
  int grid = 0;
  const int nr = vocab, kd = d;
  ChainArgs A = plan_chain_shapes(device_max_clusters(), &nr, &kd, 1, M, 0, &grid);
  PhaseArgs& P = A.ph[0];
  if (!make_map_bf16(&P.tmW, d_lm_weight, d, vocab, kTileRows) ||
      !make_map_bf16(&P.tmX, d_hidden, d, M, A.xr))
    return fail(nullptr, NLD_ERR_CUDA, "tensor map encode failed");
  P.w_rowmajor = 1;
  EpiArgs& e = P.e;
  e.kind = EPI_LMHEAD;
  e.M = M;
  e.m = M;
  e.n_rows = vocab;
  e.ssq_in = ssq;
  e.ssq_tiles = d / kTileRows;
  e.ssq_ld = M;
  e.inv_d = 1.0f / static_cast<float>(d);
  e.eps = rms_eps;
  e.lm_part = part;
  e.lm_tiles = (vocab + kTileRows - 1) / kTileRows;
  e.V = vocab;
  e.err = err;
  // rms_stats clears the error word, the chain sets it when a wait runs out, and the combine
  // then writes argmax -1 and confidence 0 for every row instead of partials never written
  cudaError_t ce = launch_rms_stats(st, d_hidden, M, d, ssq, err);
  if (ce == cudaSuccess) ce = launch_gemm_chain(st, A, grid, 2000000000ull, false);
  if (ce == cudaSuccess) ce = launch_lm_combine(st, part, M, e.lm_tiles, d_argmax_out, d_conf_out, err);
  if (ce != cudaSuccess) return fail(nullptr, NLD_ERR_CUDA, "LM-head launch failed: %s", cudaGetErrorString(ce));
  return NLD_OK;
}

size_t nld_lm_head_workspace_size(int M, int d, int vocab) {
  if (M < 1 || d < 128 || d % 128 || vocab < 1) return 0;
  return kLmErrBytes + lm_ssq_bytes(M, d) + lm_part_bytes(M, vocab);
}

nld_status nld_lm_head_argmax(const void* d_hidden, const void* d_lm_weight, int M, int d, int vocab,
                              float rms_eps, int32_t* d_argmax_out, float* d_conf_out,
                              void* d_workspace, size_t workspace_bytes, void* cuda_stream) {
  TRY(lm_head_check(d_hidden, d_lm_weight, M, d, vocab, d_argmax_out, d_conf_out));
  const size_t need = nld_lm_head_workspace_size(M, d, vocab);
  if (!d_workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(d_workspace) % 256)
    return fail(nullptr, NLD_ERR_ARG, "workspace must be 256-byte aligned and at least %zu bytes", need);
  return lm_head_launch(d_hidden, d_lm_weight, M, d, vocab, rms_eps, d_argmax_out, d_conf_out,
                        static_cast<char*>(d_workspace), static_cast<cudaStream_t>(cuda_stream));
}

// ------------------------------------------- LM head with built-in scratch (no allocation) --
// For callers that cannot allocate device memory: code running inside a framework that owns
// all device memory through its own pool (a raw cudaMalloc would bypass its budget), and
// latency-critical paths where cudaMalloc / cudaFree would synchronise the device.  The
// scratch of nld_lm_head_argmax lives in this fixed array instead; every GPU that loads the
// library holds it until the process exits.
constexpr size_t kStaticLmScratchBytes = 8u << 20;
static __device__ __align__(256) unsigned char g_lm_scratch[kStaticLmScratchBytes];

// Device address of g_lm_scratch per device (host code may not use the symbol itself as an
// address): looked up with cudaGetSymbolAddress on the first call made on each device.
static std::mutex g_lm_scratch_mu;
static void* g_lm_scratch_addr[64] = {nullptr};

size_t nld_lm_head_static_max_bytes(void) { return kStaticLmScratchBytes; }

nld_status nld_lm_head_argmax_static(const void* d_hidden, const void* d_lm_weight, int M, int d,
                                     int vocab, float rms_eps, int32_t* d_argmax_out,
                                     float* d_conf_out, void* cuda_stream) {
  TRY(lm_head_check(d_hidden, d_lm_weight, M, d, vocab, d_argmax_out, d_conf_out));
  const size_t need = nld_lm_head_workspace_size(M, d, vocab);
  if (need > kStaticLmScratchBytes)
    return fail(nullptr, NLD_ERR_ARG,
                "scratch of %zu bytes exceeds the built-in %zu bytes: 256 + M * (d/128 * 4 + ceil(vocab/128) * 16) "
                "must stay within it (use nld_lm_head_argmax with a caller workspace)",
                need, kStaticLmScratchBytes);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return fail(nullptr, NLD_ERR_CUDA, "no usable current CUDA device");
  }
  void* scratch = nullptr;
  {
    // outside stream capture the address is looked up on every call (cheap), so a device whose
    // context was reset and whose module was reloaded gets the array's new address; under
    // capture the last looked-up address is used
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(cuda_stream), &cap) != cudaSuccess) {
      cudaGetLastError();
      cap = cudaStreamCaptureStatusNone;
    }
    std::lock_guard<std::mutex> lock(g_lm_scratch_mu);
    if (!g_lm_scratch_addr[dev] || cap == cudaStreamCaptureStatusNone) {
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_lm_scratch);
      if (e != cudaSuccess || !ptr) {
        cudaGetLastError();
        return fail(nullptr, NLD_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed: %s",
                    cudaGetErrorString(e));
      }
      g_lm_scratch_addr[dev] = ptr;
    }
    scratch = g_lm_scratch_addr[dev];
  }
  return lm_head_launch(d_hidden, d_lm_weight, M, d, vocab, rms_eps, d_argmax_out, d_conf_out,
                        static_cast<char*>(scratch), static_cast<cudaStream_t>(cuda_stream));
}

// ----------------------------------------------------------------- stand-alone attention --

nld_status nld_attention(const void* d_q, const void* d_kv_pool, const int32_t* d_page_table,
                         int pages_per_seq, int n_pages, const int32_t* d_lens, int batch, int m,
                         int n_q_heads, int n_kv_heads, int head_dim, int block_size, int max_len,
                         void* d_out, void* cuda_stream) {
  if (!d_q || !d_kv_pool || !d_page_table || !d_lens || !d_out)
    return fail(nullptr, NLD_ERR_ARG, "NULL pointer argument");
  if (batch < 1 || m < 1 || n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads)
    return fail(nullptr, NLD_ERR_ARG, "bad batch/m/head counts");
  if (head_dim != 128) return fail(nullptr, NLD_ERR_UNSUPPORTED, "head_dim must be 128");
  if (block_size < 1) return fail(nullptr, NLD_ERR_ARG, "block_size must be >= 1");
  if (pages_per_seq < 1 || max_len < m || max_len > pages_per_seq * kPage)
    return fail(nullptr, NLD_ERR_ARG, "max_len outside m..pages_per_seq*64");
  if (n_pages < 1 || static_cast<long long>(n_pages) * 2 * n_kv_heads * kPage > INT32_MAX)
    return fail(nullptr, NLD_ERR_ARG, "bad pool size");
  {
    cudaError_t ae = init_kernel_attributes();
    if (ae != cudaSuccess) {
      cudaGetLastError();
      return fail(nullptr, NLD_ERR_CUDA, "setting kernel shared-memory limits failed: %s",
                  cudaGetErrorString(ae));
    }
  }
  AttnArgs a{};
  attn_plan(batch, m, n_q_heads, n_kv_heads, max_len, device_sms(), a,
            [](int S, int NW, int stages, int tc) { return attn_device_capacity(false, S, NW, stages, tc); },
            0, 0, g_attn_kernel.load(), g_attn_tile.load(), false);
  if (static_cast<long long>(batch) * a.q_tiles > 65535) return fail(nullptr, NLD_ERR_ARG, "batch*query tiles too large");
  CUtensorMap map;
  if (!make_map_bf16(&map, d_kv_pool, 128, static_cast<uint64_t>(n_pages) * 2 * n_kv_heads * kPage, kPage))
    return fail(nullptr, NLD_ERR_CUDA, "tensor map encode failed (pool)");
  a.q = d_q;
  a.out = d_out;
  a.out_ld = static_cast<size_t>(n_q_heads) * 128;
  a.m = m;
  a.Hq = n_q_heads;
  a.Hkv = n_kv_heads;
  a.hd = 128;
  a.lens = d_lens;
  a.page_table = d_page_table;
  a.pps = pages_per_seq;
  a.layer_row0 = 0;
  a.block_size = block_size;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  a.hilo = 0;   // caller's bf16 q and output
  a.err = nullptr;
  cudaError_t e = launch_attention_mma(static_cast<cudaStream_t>(cuda_stream), &map, a, batch, false);
  if (e != cudaSuccess) return fail(nullptr, NLD_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(e));
  return NLD_OK;
}

}  // extern "C"
