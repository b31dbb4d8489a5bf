// Internal declarations shared by the kernels and the host orchestration.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nld.h"

namespace nld {

constexpr int kPage = 64;          // KV page length in tokens (one attention KV tile)
constexpr int kTileRows = 128;     // GEMM weight rows per tile (tcgen05 M)
constexpr int kTileK = 64;         // GEMM K per pipeline stage (128 bytes of bf16)
constexpr int kChainSmemBudget = 227 * 1024;   // dynamic shared memory of one chain CTA (sm_100 opt-in)
constexpr int kMaxNT = 256;        // max token columns per GEMM tile (tcgen05 N)

// Epilogue kinds of the projection GEMMs.
enum EpiKind : int {
  EPI_QKV = 0,     // * 1/rms, RoPE on q/k, q -> q buffer, k/v -> paged KV cache
  EPI_RESID = 1,   // h += acc; hb = bf16(h); per-tile sum of squares of h
  EPI_SWIGLU = 2,  // * 1/rms; silu(gate) * up -> u buffer
  EPI_LMHEAD = 3,  // * 1/rms; per (token, vocab tile): max, argmax, sum exp(l - max)
  EPI_LOGITS = 4,  // * 1/rms; logits -> fp32 buffer (test hook only)
};

// Forward kinds (which tokens the embedding gathers and what the finalize step does).
enum FwdMode : int {
  FWD_AR = 0, FWD_DRAFT = 1, FWD_VERIFY = 2, FWD_DIFFUSE = 3, FWD_FILL = 4, FWD_PREFILL = 5,
  FWD_COMMIT = 6,
  FWD_FILLDIFF = 7,  // fused diffusion KV fill: [x_n, b_1..b_k, MASK x (k-1)], 2k rows
  FWD_NLDIFF = 8,    // per-sequence diffusion: flagged sequences fill, the others denoise
  FWD_NLFILL = 9,    // per-sequence diffusion: flagged sequences fill, the others keep state
  FWD_QUAD = 10      // quadratic self-speculation: verify rows + (k+1) pre-draft blocks, (k+1)^2 rows
};

// Per (token, vocab tile) partial of the LM-head reduction.
struct LmPart {
  float mx;    // max logit in the tile
  float se;    // sum over the tile of exp(l - mx)
  int idx;     // lowest vocab id attaining mx
  int pad;
};

struct EpiArgs {
  int kind;
  int M;            // tokens in this forward (columns)
  int m;            // rows per sequence
  int n_rows;       // valid weight rows (GEMM outputs)
  // RMSNorm of the GEMM input: 1/rms[tok] = rsqrt(sum_t ssq_in[t*ld + tok] / d + eps)
  const float* ssq_in;
  int ssq_tiles;
  int ssq_ld;
  float inv_d;
  float eps;
  // EPI_QKV
  void* q_out;      // [M, Hq, hd]
  int Hq, Hkv, hd;
  void* kv_layer;   // pool base of this layer: [n_pages][2][Hkv][64][hd]
  const int* page_table;  // [batch, pps]
  int pps;
  const int* lens;  // [batch]
  const float2* rope;  // [kv_cap, hd/2] (cos, sin)
  int kv_cap;
  // EPI_RESID
  float* h;         // [M, d]
  void* hb;         // [M, d]
  float* ssq_out;   // [d/128, ssq_ld]
  int d;
  // EPI_SWIGLU
  void* u_out;      // [M, F]
  int F;
  // EPI_LMHEAD / EPI_LOGITS
  LmPart* lm_part;  // [M, lm_tiles]
  int lm_tiles;
  float* logits;    // [M, V]
  int V;
  int hilo;         // bf16 storage: hb / u written as (hi, lo) row pairs [2M, ld], q in fp32
  int quad_k;       // quadratic self-speculation forward with block k: RoPE positions of the
                    // pre-draft rows differ from their KV slots (0 = every other forward)
  int* err;
};

// Entries of a chain launch's profiling trace: 16 per CTA (grid <= 148), then CTA 0's
// per-iteration pipeline stamps (4 kinds x 64).
constexpr int kChainTraceEntries = 148 * 16 + 4 * 64;

// One projection of a chain launch.
constexpr int kMaxPhases = 4;
struct alignas(64) PhaseArgs {
  CUtensorMap tmW;  // row-major weights (w_rowmajor): box {64, 128} at (k * 64, row)
  CUtensorMap tmX;  // activations [M_max, K], box {64, NT}
  const void* W;    // pre-tiled weights (w_rowmajor == 0): block (row tile r, k-tile kt) is the
                    // 16 KB swizzled shared-memory image at byte offset (r * KT + kt) * 16384
  EpiArgs e;
  int tok_tiles, row_tiles, KT;
  int s;            // ranks of a cluster splitting each tile's K range (divides CS)
  int ks;           // k-iterations per rank
  int w_rowmajor;   // 1: tmW views a plain row-major [n_rows, K] matrix (box {64, 128} at
                    // (k*64, row)); 0: the pre-tiled layout
  int x3d;          // 1: tmX views the activations as [K/64 blocks][rows][64] with box
                    // {64, xr, kps}: one load brings a stage's kps k-tiles of a token tile
                    // (rows past the tensor fill with zeros); 0: 2D [rows, K], box {64, xr}
};

// One phase of the next chain launch, as far as the L2 warm-up needs it.
struct WarmPhase {
  const void* W;    // pre-tiled weights of that phase
  int s, tok_tiles, ks, KT, tiles;
  int boxes;        // 16 KB weight boxes to prefetch per CTA (0 = none)
};

// A persistent launch running nph projections in order, separated by grid-wide arrivals.
struct alignas(64) ChainArgs {
  PhaseArgs ph[kMaxPhases];
  int nph;
  int CS;           // CTAs per cluster
  int NT;           // tokens per tile (multiple of 16; MMA N = NT << hilo <= 256)
  int stages;       // shared-memory ring depth
  int kps;          // k-tiles (of 64) per stage: one barrier round trip moves kps x 16 KB of weights
  int xr;           // activation rows loaded per k-tile of a token tile: the tile's rows (2 per
                    // token with hilo) rounded up to 8 (<= MMA N); the MMA reads past them into
                    // padding columns that the epilogue never uses
  int slots;        // split-K slot area: max over split phases of s * ceil(NT/16 / s) chunks
  int hilo;         // activation rows come in (hi, lo) pairs: MMA N = 2 NT, chunk sums of pairs
  uint32_t tmem_cols;   // power of two >= 2 * MMA N
  unsigned* bar;    // [kMaxPhases] phase-boundary arrival counters + exit counter (last slot);
                    // zero before the launch, left zero by it
  unsigned long long* trace;   // optional per-CTA phase timestamps (profiling hook), or null
  int boundary_pf;  // weight boxes each CTA prefetches into L2 while it waits at a phase boundary
  int pf_stages;    // L2 run-ahead: stages between a weight prefetch and its load (0 = off)
  int dbg_skip_arrive;   // test hook: CTA 0 withholds its phase-0 arrival, so every wait on that
                         // counter runs into its time limit (the failure-detection test)
  // the next chain launch on the stream: before exiting, each CTA prefetches into L2 the first
  // weight boxes that the CTA of the same index loads in that launch's first two phases, so HBM
  // streams them while the kernels in between (attention) run
  int next_valid;
  int next_CS, next_grid;
  WarmPhase next[2];
};

struct AttnArgs {
  const void* q;        // [M, Hq, hd]
  void* out;            // [M, Hq, hd] rows out_ld elements apart (tensor-core path)
  size_t out_ld;
  const void* pool;     // SIMT path: pool base of this layer
  int m, Hq, Hkv, G, hd;
  const int* lens;
  const int* page_table;
  int pps;
  int layer_row0;       // row of this layer's first page in the 2D pool view
  int block_size;
  int causal_rows;      // the first causal_rows rows of each sequence are strictly causal and
                        // the blocks of block_size start after them (fused diffusion fill)
  const int* causal_seq;  // optional [batch]: nonzero makes all m rows of that sequence causal
  int QT, q_tiles, rows, S, NW;   // S = KV splits = cluster size (1..8)
  int min_tiles;        // KV tiles a split takes at least (1..)
  int stages;           // K/V ring depth of the tensor-core path (2 or 3)
  int tc;               // 2 / 4: the tcgen05 kernel (query tiles of <= 128 rows) with 2 / 4
                        // softmax threads per row; 0: mma.sync
  int tc_tile;          // tcgen05: keys per KV tile, 64 or 128
  float scale_log2;     // log2(e) / sqrt(hd)
  int hilo;             // tensor-core path: q fp32 [M, Hq, hd], out (hi, lo) bf16 rows [2M, Hq, hd]
  int quad_k;           // quadratic self-speculation forward with block k (0 = off): rows 0..k are
                        // causal; pre-draft row k+1+a*k+j sees the prefix, rows 0..a and its block
  unsigned long long* trace;   // optional per-CTA timestamps (profiling hook), or null
  int* err;
};

// ---- host-side launchers (each returns cudaError_t of the launch) -----------------------
cudaError_t launch_gemm_chain(cudaStream_t st, const ChainArgs& A, int grid, uint64_t timeout_ns,
                              bool pdl);
size_t gemm_chain_smem_bytes(int NT, int nn, int xr, int kps, int stages, int CS, int slots);
int gemm_chain_max_stages();
int gemm_tc_max_clusters(int split, size_t smem, int sms);
cudaError_t launch_gemm_simt(cudaStream_t st, const float* W, const float* X, int n_rows, int K,
                             int M, const EpiArgs& e, bool pdl);
cudaError_t launch_attention_mma(cudaStream_t st, const CUtensorMap* tmKV, const AttnArgs& a,
                                 int batch, bool pdl);
cudaError_t launch_attention_simt(cudaStream_t st, const AttnArgs& a, int batch, bool f32,
                                  int max_kv, bool pdl);

struct EmbedArgs {
  const void* E;        // [V+1, d]
  int d, V, m, mode, k;
  const int* pending; const int* draft; const int* blk;
  const int* prompt; int prompt_len; int chunk0;
  const int* plens;     // prefill: [batch] prompt lengths (rows at or past plens[b]-1 are padding)
  const int* lens;
  float* h; void* hb; float* ssq; int ssq_ld;
  int hilo;             // bf16: hb rows in (hi, lo) pairs (the embedding row, then zeros)
  int* err;
};
cudaError_t launch_embed(cudaStream_t st, const EmbedArgs& a, int M, bool bf16, bool pdl);

struct FinalizeArgs {
  int mode, m, k, V, lm_tiles;
  const LmPart* lm_part;
  int* lens; int* pending; int* draft; int* verify; int* blk;
  int* tokens_out; int* ncommit_out; const int* force; float* conf_out; int* block_out;
  float threshold;
  int* incomplete;      // diffusion: count of sequences whose block is still open
  const int* prompt; int prompt_len; int chunk;   // prefill
  const int* plens;     // prefill: [batch] prompt lengths (<= prompt_len, the row stride)
  int* pending_out;     // prefill: [batch] the pending token of each sequence, or null
  int commit;           // 0 = only record argmaxes (test hook)
  int kv_cap;
  int* err;
  int* fillnext;        // per-sequence diffusion: [batch] fill flags (read and updated)
  int* state_out;       // per-sequence diffusion: 0 open, 1 completed now, 2 filled now
};
cudaError_t launch_finalize(cudaStream_t st, const FinalizeArgs& a, int batch, bool pdl);

cudaError_t launch_repack(cudaStream_t st, void* dst, const void* src, const int* row_map,
                          int n_rows, int K, const void* gamma, bool bf16, bool tiled);
cudaError_t launch_fill_i32(cudaStream_t st, int* p, int value, int n);
// LoRA drafter: fp32 partials zp [lora_n_ks][M][r] of z = A att, then h += scale * B z on
// the rows t with t mod m >= causal_rows of sequences b = t / m whose causal_seq flag (if
// given) is zero.  With hilo, att holds (hi, lo) bf16 row pairs [2M, qd] whose sums are the
// attention output, and z stays fp32; otherwise z is rounded to the activation type.
// A [r, qd], B [d, r] row-major; 8 <= r <= 256, r % 8 == 0; qd a multiple of 8.
int lora_n_ks(int qd, bool bf16);
// The drafter's z = scale * A att of the bf16 (hi, lo) forward, written as (hi, lo) bf16 into
// columns qd..qd+r of the rows of zout (row pitch ld; rows 2t, 2t+1), where the O projection of
// the layer chain reads it as r more K columns against scale-free B (the folded adapter).
// cnt: [ceil(r/16) * ceil(M/32)] zero counters (left zero).
cudaError_t launch_lora_z(cudaStream_t st, const void* A, const void* att, size_t att_ld, float* zp,
                          int* cnt, void* zout, size_t ld, int M, int qd, int r, float scale, int m,
                          int causal_rows, const int* causal_seq, bool pdl);
cudaError_t launch_lora(cudaStream_t st, const void* A, const void* B, const void* att, float* zp,
                        float* h, int M, int qd, int d, int r, float scale, int m, int causal_rows,
                        const int* causal_seq, bool bf16, bool hilo, bool pdl);
// Per 128-column tile sums of squares of bf16 rows h [M, d] into ssq [d/128, M]; zeroes *err.
cudaError_t launch_rms_stats(cudaStream_t st, const void* h, int M, int d, float* ssq, int* err);
// Per token: argmax (lowest id on ties) and largest softmax probability from LM-head partials;
// argmax -1 and confidence 0 when *err is set (the partials were not all written).
cudaError_t launch_lm_combine(cudaStream_t st, const LmPart* part, int M, int tiles, int* argmax,
                              float* conf, const int* err);

}  // namespace nld
