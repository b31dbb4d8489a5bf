// Per-forward small kernels: embedding gather (builds each mode's input block on the device),
// the finalize step after the LM head (argmax/confidence combine over vocab tiles and the
// mode's state update: drafts, AR commit, greedy acceptance, diffusion commit in lockstep,
// fused or per-sequence form, KV-fill and prefill bookkeeping), the optional LoRA drafter's two
// kernels, weight repacking and fills.
#include <algorithm>
#include <climits>

#include "common.cuh"

namespace nld {

constexpr int kFinalizeThreads = 1024;   // one warp per LM-head row of a sequence (m <= 64)

// ------------------------------------------------------------------------------ embedding --
// Input block of each forward (shifted prediction; the pending token x_n sits at position n):
//   AR      [x_n]                         DRAFT   [x_n, MASK x (k-1)]
//   VERIFY  [x_n, d_1..d_k]               DIFFUSE / FILL [x_n, b_1..b_{k-1}]
//   PREFILL prompt[chunk0 .. chunk0+m-1]
// h = E[token] (fp32 residual), hb = the GEMM operand copy, and per 128-column tile the sum of
// squares of h (the RMSNorm statistics the next GEMM epilogue turns into 1/rms).
template <typename T>
__global__ void __launch_bounds__(256) embed_kernel(const EmbedArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  const int b = t / a.m, i = t - b * a.m;
  int id;
  switch (a.mode) {
    case FWD_PREFILL:
      // rows at or past the sequence's own last prompt position are padding of a ragged batch
      // (their KV rows lie past its length and are overwritten before any query sees them)
      id = (a.plens && a.chunk0 + i >= a.plens[b] - 1)
               ? 0
               : a.prompt[static_cast<size_t>(b) * a.prompt_len + a.chunk0 + i];
      break;
    case FWD_AR: id = a.pending[b]; break;
    case FWD_DRAFT: id = (i == 0) ? a.pending[b] : a.V; break;
    case FWD_VERIFY: id = (i == 0) ? a.pending[b] : a.draft[b * a.k + i - 1]; break;
    case FWD_FILLDIFF:   // the complete block (causal rows), then b_k and k-1 masks
      id = (i == 0) ? a.pending[b] : (i <= a.k ? a.blk[b * a.k + i - 1] : a.V);
      break;
    case FWD_QUAD:       // verify rows [x_n, d_1..d_k], then (k+1) pre-draft blocks of masks
      id = (i == 0) ? a.pending[b] : (i <= a.k ? a.draft[b * a.k + i - 1] : a.V);
      break;
    default: id = (i == 0) ? a.pending[b] : a.blk[b * a.k + i - 1]; break;
  }
  if (id < 0 || id > a.V) {
    set_err(a.err, NLD_DEVERR_TOKEN);
    id = 0;
  }
  const T* row = static_cast<const T*>(a.E) + static_cast<size_t>(id) * a.d;
  float* h = a.h + static_cast<size_t>(t) * a.d;
  // bf16 operands: the (hi, lo) row pair of token t; an embedding row is exact in bf16, so lo = 0
  const bool hl = (sizeof(T) == 2) && a.hilo;
  T* hb = static_cast<T*>(a.hb) + static_cast<size_t>(hl ? 2 * t : t) * a.d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = a.d / kTileRows;
  for (int tile = warp; tile < ntiles; tile += 8) {
    float sq = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = tile * kTileRows + lane * 4 + q;
      const float v = to_f32<T>(row[c]);
      h[c] = v;
      hb[c] = row[c];
      if (hl) hb[a.d + c] = from_f32<T>(0.f);
      sq += v * v;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) a.ssq[static_cast<size_t>(tile) * a.ssq_ld + t] = sq;
  }
}

cudaError_t launch_embed(cudaStream_t st, const EmbedArgs& a, int M, bool bf16, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (bf16) return cudaLaunchKernelEx(&cfg, embed_kernel<__nv_bfloat16>, a);
  return cudaLaunchKernelEx(&cfg, embed_kernel<float>, a);
}

// ------------------------------------------------------------------------------- finalize --
// One CTA per sequence.  For forwards with an LM head, warp w combines rows w, w+8, ... over
// all vocab tiles: global max (lowest id on ties) and sum_t se_t * exp(mx_t - max), whose
// inverse is the largest softmax probability (the confidence).
// Merge of two LM-head partials (max, sum of exp(l - max), lowest argmax) into a.
NLD_DEV void lm_merge(float& mx, float& se, int& ix, float bmx, float bse, int bix) {
  if (bmx == -INFINITY) return;
  if (bmx > mx || (bmx == mx && bix < ix)) {
    se = bse + ((mx == -INFINITY) ? 0.f : se * expf(mx - bmx));
    mx = bmx;
    ix = bix;
  } else {
    se += bse * expf(bmx - mx);
  }
}

// Combine the LM-head partials of row `row` of sequence b (one warp): argmax (lowest id on ties)
// and confidence, valid in every lane.
NLD_DEV void combine_row(const FinalizeArgs& a, int b, int row, int lane, int& ix_out, float& conf_out) {
  const LmPart* part = a.lm_part + static_cast<size_t>(b * a.m + row) * a.lm_tiles;
  float mx = -INFINITY, se = 0.f;
  int ix = INT_MAX;
  for (int t0 = lane; t0 < a.lm_tiles; t0 += 32 * 8) {
    LmPart p[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int t = t0 + 32 * u;
      if (t < a.lm_tiles) {
        p[u] = part[t];
      } else {
        p[u].mx = -INFINITY;
        p[u].se = 0.f;
        p[u].idx = INT_MAX;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) lm_merge(mx, se, ix, p[u].mx, p[u].se, p[u].idx);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mx, off);
    const float os = __shfl_xor_sync(0xffffffffu, se, off);
    const int oi = __shfl_xor_sync(0xffffffffu, ix, off);
    lm_merge(mx, se, ix, om, os, oi);
  }
  ix_out = ix;
  conf_out = 1.0f / se;
}

// Quadratic self-speculation round (one CTA per sequence): the verify rows 0..k give v_1..v_{k+1};
// the round commits as the linear round does (greedy longest matching prefix, c = a+1 tokens
// d_1..d_a, v_{a+1}); the next drafts are the argmaxes of pre-draft block a (rows
// k+1+a*k .. k+1+a*k+k-1), the block whose rows assumed exactly this outcome.
NLD_DEV void finalize_quad(const FinalizeArgs& a, int b, int warp, int lane, int* s_arg) {
  const int k = a.k;
  __shared__ int s_c;
  for (int i = warp; i <= k; i += kFinalizeThreads / 32) {
    int ix;
    float cf;
    combine_row(a, b, i, lane, ix, cf);
    if (lane == 0) s_arg[i] = ix;
  }
  __syncthreads();
  if (warp == 0) {
    const bool match = (lane < k) ? (a.draft[b * k + lane] == s_arg[lane]) : true;
    const unsigned bal = __ballot_sync(0xffffffffu, match);
    const int acc = min((bal == 0xffffffffu) ? 32 : (__ffs(~bal) - 1), k);
    const int c = acc + 1;
    for (int j = lane; j < k + 1; j += 32) {
      const int v = (j < c - 1) ? a.draft[b * k + j] : (j == c - 1 ? s_arg[j] : -1);
      if (a.tokens_out) a.tokens_out[b * (k + 1) + j] = v;
      a.verify[b * (k + 1) + j] = s_arg[j];
    }
    __syncwarp();
    if (lane == 0) {
      if (a.ncommit_out) a.ncommit_out[b] = c;
      a.lens[b] += c;
      a.pending[b] = s_arg[c - 1];
      s_c = c;
    }
  }
  __syncthreads();
  const int r0 = k + 1 + (s_c - 1) * k;
  for (int i = warp; i < k; i += kFinalizeThreads / 32) {
    int ix;
    float cf;
    combine_row(a, b, r0 + i, lane, ix, cf);
    if (lane == 0) a.draft[b * k + i] = ix;   // the old drafts were read by warp 0 above
  }
}

__global__ void __launch_bounds__(kFinalizeThreads) finalize_kernel(const FinalizeArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int s_arg[64];
  __shared__ float s_conf[64];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.mode == FWD_QUAD) {
    finalize_quad(a, b, warp, lane, s_arg);
    return;
  }
  const bool lm = (a.mode == FWD_AR || a.mode == FWD_DRAFT || a.mode == FWD_VERIFY ||
                   a.mode == FWD_DIFFUSE || a.mode == FWD_FILLDIFF || a.mode == FWD_NLDIFF);
  if (lm) {
    // one warp per row; one pass over the row's vocab tiles with 8 loads in flight per lane,
    // merging (max, sum exp, argmax) online, then across the warp
    for (int i = warp; i < a.m; i += kFinalizeThreads / 32) {
      int ix;
      float cf;
      combine_row(a, b, i, lane, ix, cf);
      if (lane == 0) {
        s_arg[i] = ix;
        s_conf[i] = cf;
      }
    }
    __syncthreads();
  }
  if (warp != 0) return;
  const int k = a.k;
  switch (a.mode) {
    case FWD_AR: {
      if (lane == 0) {
        const int tok = s_arg[0];
        if (a.commit) {
          a.pending[b] = tok;
          a.lens[b] += 1;
          if (a.tokens_out) a.tokens_out[b] = tok;
        }
      }
    } break;
    case FWD_DRAFT: {
      for (int i = lane; i < k; i += 32) a.draft[b * k + i] = s_arg[i];
    } break;
    case FWD_VERIFY: {
      for (int i = lane; i < k + 1; i += 32) a.verify[b * (k + 1) + i] = s_arg[i];
    } break;
    case FWD_COMMIT: {
      // greedy longest matching prefix: a = index of the first mismatch among d_i == v_i
      const bool match = (lane < k) ? (a.draft[b * k + lane] == a.verify[b * (k + 1) + lane]) : true;
      const unsigned bal = __ballot_sync(0xffffffffu, match);
      int acc = (bal == 0xffffffffu) ? 32 : (__ffs(~bal) - 1);
      acc = min(acc, k);
      int c = acc + 1;
      if (a.force) {
        c = a.force[b];
        if (c < 1 || c > k + 1) {
          if (lane == 0) set_err(a.err, NLD_DEVERR_TOKEN);
          c = max(1, min(c, k + 1));
        }
      }
      for (int j = lane; j < k + 1; j += 32) {
        int v;
        if (j < c - 1) v = a.draft[b * k + j];
        else if (j == c - 1) v = a.verify[b * (k + 1) + j];
        else v = -1;
        if (a.tokens_out) a.tokens_out[b * (k + 1) + j] = v;
      }
      __syncwarp();
      if (lane == 0) {
        if (a.ncommit_out) a.ncommit_out[b] = c;
        a.lens[b] += c;
        a.pending[b] = a.verify[b * (k + 1) + c - 1];
      }
    } break;
    case FWD_NLFILL:
    case FWD_NLDIFF:
    case FWD_FILLDIFF:
    case FWD_DIFFUSE: {
      // FWD_NLDIFF / FWD_NLFILL (per-sequence diffusion): a sequence flagged in fillnext ran its
      // causal KV fill in this forward (all its rows causal): len += k, pending = b_k, a fresh
      // block of masks.  The others denoise (FWD_NLFILL: keep their state).
      const bool nl = (a.mode == FWD_NLDIFF || a.mode == FWD_NLFILL);
      if (nl && a.fillnext[b] != 0) {
        const int last = a.blk[b * k + k - 1];
        __syncwarp();
        for (int i = lane; i < k; i += 32) {
          a.blk[b * k + i] = a.V;
          if (a.block_out) a.block_out[b * k + i] = a.V;
          if (a.conf_out) a.conf_out[b * k + i] = 0.f;
        }
        if (lane == 0) {
          a.lens[b] += k;
          a.pending[b] = last;
          a.fillnext[b] = 0;
          if (a.ncommit_out) a.ncommit_out[b] = 0;
          if (a.state_out) a.state_out[b] = 2;
        }
        break;
      }
      if (a.mode == FWD_NLFILL) break;
      // FWD_FILLDIFF: the complete block's KV rows were written by this forward's first k
      // (causal) rows: len += k, pending = b_k, and the new block (all masks) is denoised by
      // the last k rows
      const bool fused = (a.mode == FWD_FILLDIFF);
      const int row0 = fused ? k : 0;
      if (fused) {
        const int last = a.blk[b * k + k - 1];
        __syncwarp();
        if (a.commit)
          for (int i = lane; i < k; i += 32) a.blk[b * k + i] = a.V;
        __syncwarp();
        if (lane == 0 && a.commit) {
          a.lens[b] += k;
          a.pending[b] = last;
        }
      }
      // confidence-threshold commit among open slots; at least one (the most confident)
      const bool valid = lane < k;
      const int cur = valid ? (fused ? a.V : a.blk[b * k + lane]) : 0;
      const bool masked = valid && (cur == a.V);
      const float conf = valid ? s_conf[row0 + lane] : 0.f;
      const int tok = valid ? s_arg[row0 + lane] : 0;
      bool pick = masked && (conf >= a.threshold);
      const unsigned any_pick = __ballot_sync(0xffffffffu, pick);
      const unsigned any_mask = __ballot_sync(0xffffffffu, masked);
      if (any_pick == 0u && any_mask != 0u) {
        float best = masked ? conf : -1.f;
        int bi = masked ? lane : 64;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
          if (ob > best || (ob == best && oi < bi)) {
            best = ob;
            bi = oi;
          }
        }
        pick = (lane == bi);
      }
      const unsigned picked = __ballot_sync(0xffffffffu, pick);
      const unsigned still_open = __ballot_sync(0xffffffffu, masked && !pick);
      const int nb = pick ? tok : cur;
      if (valid) {
        if (a.commit) a.blk[b * k + lane] = nb;
        if (a.conf_out) a.conf_out[b * k + lane] = conf;
        if (a.block_out) a.block_out[b * k + lane] = nb;
      }
      if (lane == 0) {
        if (a.ncommit_out) a.ncommit_out[b] = __popc(picked);
        if (a.commit && still_open != 0u && a.incomplete) atomicAdd(a.incomplete, 1);
        if (nl) {   // a completed block is filled by this sequence's next step
          if (a.commit) a.fillnext[b] = (still_open == 0u) ? 1 : 0;
          if (a.state_out) a.state_out[b] = (still_open == 0u) ? 1 : 0;
        }
      }
    } break;
    case FWD_FILL: {
      const int last = a.blk[b * k + k - 1];
      __syncwarp();
      for (int i = lane; i < k; i += 32) a.blk[b * k + i] = a.V;
      if (lane == 0) {
        a.lens[b] += k;
        a.pending[b] = last;
      }
    } break;
    case FWD_PREFILL: {
      if (lane == 0) {
        if (a.prompt) {
          // last chunk: the sequence's own length and pending token
          int plen = a.plens ? a.plens[b] : a.prompt_len;
          if (plen < 1 || plen > a.prompt_len) {
            set_err(a.err, NLD_DEVERR_TOKEN);
            plen = max(1, min(plen, a.prompt_len));
          }
          const int tok = a.prompt[static_cast<size_t>(b) * a.prompt_len + plen - 1];
          a.lens[b] = plen - 1;
          a.pending[b] = tok;
          if (a.pending_out) a.pending_out[b] = tok;
        } else {
          a.lens[b] += a.chunk;
        }
      }
    } break;
    default:
      break;
  }
}

cudaError_t launch_finalize(cudaStream_t st, const FinalizeArgs& a, int batch, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch);
  cfg.blockDim = dim3(kFinalizeThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, finalize_kernel, a);
}

// ------------------------------------------------------------------------- LoRA drafter --
// Low-rank delta on o_proj in the block-bidirectional (drafter) forwards: h += scale * B (A att),
// added to the residual before the layer chain adds W_o att.  A [r, qd], B [d, r] row-major
// (the caller's layout); rank r a multiple of 8.  Two launches, both latency-bound at decode
// sizes (1 MB of adapter weights per matrix at r 128, d 4096), so every global load of a CTA
// is a 16-byte vector load issued before any arithmetic.
//
// z partials: CTA (jg, ks, tg) takes 16 adapter rows x one 512-byte column slice of qd x 32
// tokens, stages the A and att slices in shared memory (rows padded so that the per-token
// reads of a warp hit distinct banks) and writes zp[ks][t][j] = sum over its slice (fp32).
// The slices are summed in a fixed order by lora_up: deterministic, no atomics.
constexpr int kLoraJ = 16, kLoraT = 32, kLoraThreads = 256;
template <typename T> struct LoraCols { static constexpr int n = 512 / sizeof(T); };

// With a counter array (the folded form, bf16 (hi, lo) forwards only): the CTA that completes a
// (16 adapter rows, 32 tokens) block last sums its slices in slice order (deterministic), scales
// by `scale` and writes z as (hi, lo) bf16 pairs into columns qd + j of rows 2t, 2t+1 of zout
// (pitch ld), zero for rows that are not drafter rows (as lora_up skips them).
struct LoraFinal {
  int* cnt;           // [gridDim.x * gridDim.z] zero counters, left zero
  __nv_bfloat16* zout;
  size_t ld;
  float scale;
  int m, causal_rows;
  const int* causal_seq;
};

template <typename T, bool kHiLo>
__global__ void __launch_bounds__(kLoraThreads) lora_down_kernel(const T* A, const T* att, size_t att_ld,
                                                                 float* zp, int M, int qd, int r,
                                                                 const LoraFinal fin) {
  constexpr int C = LoraCols<T>::n, LD = C + 2, V = 16 / sizeof(T);
  constexpr int kXRows = kHiLo ? 2 * kLoraT : kLoraT;   // with hi/lo: rows 2t, 2t+1 per token
  __shared__ __align__(16) T sA[kLoraJ][LD];
  __shared__ __align__(16) T sX[kXRows][LD];
  pdl_wait();
  pdl_launch_dependents();
  const int j0 = blockIdx.x * kLoraJ, c0 = blockIdx.y * C, t0 = blockIdx.z * kLoraT;
  // stage: 16 + 32 (64 with hi/lo) rows of C/V vectors; out-of-range rows and columns read as zero
  constexpr int kVecRow = C / V, kVecs = (kLoraJ + kXRows) * kVecRow;
  uint4 v[(kVecs + kLoraThreads - 1) / kLoraThreads];
#pragma unroll
  for (int u = 0; u < (kVecs + kLoraThreads - 1) / kLoraThreads; ++u) {
    const int e = u * kLoraThreads + threadIdx.x;
    const int row = e / kVecRow, c = c0 + (e % kVecRow) * V;
    v[u] = make_uint4(0, 0, 0, 0);
    if (e < kVecs && c < qd) {
      if (row < kLoraJ) {
        if (j0 + row < r) v[u] = *reinterpret_cast<const uint4*>(A + static_cast<size_t>(j0 + row) * qd + c);
      } else if (((row - kLoraJ) >> (kHiLo ? 1 : 0)) + t0 < M) {
        // att row index: token t0 + i (plain) or row 2 t0 + i of the (hi, lo) pairs
        const size_t arow = (kHiLo ? 2 * static_cast<size_t>(t0) : static_cast<size_t>(t0)) + (row - kLoraJ);
        v[u] = *reinterpret_cast<const uint4*>(att + arow * att_ld + c);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < (kVecs + kLoraThreads - 1) / kLoraThreads; ++u) {
    const int e = u * kLoraThreads + threadIdx.x;
    if (e < kVecs) {
      const int row = e / kVecRow, cc = (e % kVecRow) * V;
      T* dst = (row < kLoraJ) ? &sA[row][cc] : &sX[row - kLoraJ][cc];
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) reinterpret_cast<uint32_t*>(dst)[q] = w[q];   // rows 4-byte aligned
    }
  }
  __syncthreads();
  // lane = token, warp = adapter rows 2w, 2w+1
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
  for (int c = 0; c < C; c += 2) {
    float x0, x1, p0, p1, q0, q1;
    if constexpr (sizeof(T) == 2) {
      float2 xx;
      if constexpr (kHiLo) {
        const float2 xh = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sX[2 * lane][c]));
        const float2 xl = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sX[2 * lane + 1][c]));
        xx = make_float2(xh.x + xl.x, xh.y + xl.y);
      } else {
        xx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sX[lane][c]));
      }
      const float2 pp = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sA[2 * w][c]));
      const float2 qq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&sA[2 * w + 1][c]));
      x0 = xx.x; x1 = xx.y; p0 = pp.x; p1 = pp.y; q0 = qq.x; q1 = qq.y;
    } else {
      const float2 xx = *reinterpret_cast<const float2*>(&sX[lane][c]);
      const float2 pp = *reinterpret_cast<const float2*>(&sA[2 * w][c]);
      const float2 qq = *reinterpret_cast<const float2*>(&sA[2 * w + 1][c]);
      x0 = xx.x; x1 = xx.y; p0 = pp.x; p1 = pp.y; q0 = qq.x; q1 = qq.y;
    }
    a0 = fmaf(p0, x0, a0);
    a0 = fmaf(p1, x1, a0);
    a1 = fmaf(q0, x0, a1);
    a1 = fmaf(q1, x1, a1);
  }
  const int t = t0 + lane, j = j0 + 2 * w;
  if (t < M) {
    float* out = zp + (static_cast<size_t>(blockIdx.y) * M + t) * r;
    if (j < r) out[j] = a0;
    if (j + 1 < r) out[j + 1] = a1;
  }
  if (fin.cnt == nullptr) return;
  // folded form: the block's last slice CTA (release/acquire through the counter) sums
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  int* cnt = fin.cnt + blockIdx.x * gridDim.z + blockIdx.z;
  if (threadIdx.x == 0) s_last = (atomicAdd(cnt, 1) == static_cast<int>(gridDim.y) - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int e = threadIdx.x; e < kLoraJ * kLoraT; e += kLoraThreads) {
    const int jj = j0 + e % kLoraJ, tt = t0 + e / kLoraJ;
    if (jj >= r || tt >= M) continue;
    float acc = 0.f;
    for (int ks = 0; ks < static_cast<int>(gridDim.y); ++ks)   // slice order; other CTAs' writes: not L1
      acc += __ldcg(zp + (static_cast<size_t>(ks) * M + tt) * r + jj);
    const bool drafter = (tt % fin.m) >= fin.causal_rows && !(fin.causal_seq && fin.causal_seq[tt / fin.m]);
    __nv_bfloat16 hi, lo;
    split_bf16(drafter ? fin.scale * acc : 0.f, hi, lo);
    fin.zout[(2 * static_cast<size_t>(tt)) * fin.ld + qd + jj] = hi;
    fin.zout[(2 * static_cast<size_t>(tt) + 1) * fin.ld + qd + jj] = lo;
  }
  if (threadIdx.x == 0) *cnt = 0;   // every CTA of the block has arrived
}

// h[t][i] += scale * sum_j B[i][j] z[t][j], z = the activation-type rounding of the summed
// partials.  A CTA per 128 outputs i and 8 tokens; thread i reads its own row of B in 64-column
// chunks of 16-byte loads (all issued before the chunk's arithmetic); z rows broadcast from
// shared memory.  Rows t with t mod m < causal_rows (the fused fill's causal rows) and the
// rows of sequences flagged in causal_seq (a per-sequence fill) are not drafter rows and keep h
// unchanged.
template <typename T, bool kHiLo>
__global__ void __launch_bounds__(128) lora_up_kernel(const T* B, const float* zp, float* h, int M,
                                                      int d, int r, int n_ks, float scale, int m,
                                                      int causal_rows, const int* causal_seq) {
  constexpr int kChunk = 64, V = 16 / sizeof(T), kLd = kChunk / V;
  __shared__ __align__(16) float s_z[8][256];
  pdl_wait();
  pdl_launch_dependents();
  const int i = blockIdx.x * 128 + threadIdx.x;
  const int t0 = blockIdx.y * 8;
  const int nt = min(8, M - t0);
  // the 8 token rows of a partial are contiguous (8*r floats): element e = tt*r + j.  Four
  // slices' loads of all of a thread's elements are issued before any is summed (64 loads in
  // flight), and the sums run in slice order (deterministic)
  constexpr int kQ = 8 * 256 / 128, kS = 4;
  float za[kQ];
#pragma unroll
  for (int q = 0; q < kQ; ++q) za[q] = 0.f;
  for (int ks0 = 0; ks0 < n_ks; ks0 += kS) {
    float t[kS][kQ];
#pragma unroll
    for (int u = 0; u < kS; ++u) {
      const float* zk = zp + (static_cast<size_t>(ks0 + u) * M + t0) * r;
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const int e = q * 128 + threadIdx.x;
        t[u][q] = (ks0 + u < n_ks && e < nt * r) ? zk[e] : 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kS; ++u)
#pragma unroll
      for (int q = 0; q < kQ; ++q) za[q] += t[u][q];
  }
#pragma unroll
  for (int q = 0; q < kQ; ++q) {
    const int e = q * 128 + threadIdx.x;
    if (e < 8 * r) s_z[e / r][e % r] = kHiLo ? za[q] : to_f32<T>(from_f32<T>(za[q]));   // rows >= nt: zero
  }
  __syncthreads();
  if (i >= d) return;
  float acc[8];
#pragma unroll
  for (int tt = 0; tt < 8; ++tt) acc[tt] = 0.f;
  const T* brow = B + static_cast<size_t>(i) * r;
  for (int j0 = 0; j0 < r; j0 += kChunk) {
    uint4 v[kLd];
#pragma unroll
    for (int u = 0; u < kLd; ++u)
      v[u] = (j0 + u * V < r) ? *reinterpret_cast<const uint4*>(brow + j0 + u * V) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < kLd; ++u) {
      const T* bv = reinterpret_cast<const T*>(&v[u]);
      const int jb = j0 + u * V;
      if (jb >= r) break;
#pragma unroll
      for (int q = 0; q < V; q += 4) {
        const float b0 = to_f32<T>(bv[q]), b1 = to_f32<T>(bv[q + 1]);
        const float b2 = to_f32<T>(bv[q + 2]), b3 = to_f32<T>(bv[q + 3]);
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          const float4 z4 = *reinterpret_cast<const float4*>(&s_z[tt][jb + q]);
          acc[tt] = fmaf(b0, z4.x, acc[tt]);
          acc[tt] = fmaf(b1, z4.y, acc[tt]);
          acc[tt] = fmaf(b2, z4.z, acc[tt]);
          acc[tt] = fmaf(b3, z4.w, acc[tt]);
        }
      }
    }
  }
  for (int tt = 0; tt < nt; ++tt)
    if ((t0 + tt) % m >= causal_rows && !(causal_seq && causal_seq[(t0 + tt) / m]))
      h[static_cast<size_t>(t0 + tt) * d + i] += scale * acc[tt];
}

int lora_n_ks(int qd, bool bf16) {
  const int C = bf16 ? LoraCols<__nv_bfloat16>::n : LoraCols<float>::n;
  return (qd + C - 1) / C;
}

cudaError_t launch_lora(cudaStream_t st, const void* A, const void* B, const void* att, float* zp,
                        float* h, int M, int qd, int d, int r, float scale, int m, int causal_rows,
                        const int* causal_seq, bool bf16, bool hilo, bool pdl) {
  if (r < 8 || r > 256 || r % 8 || M < 1) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const int n_ks = lora_n_ks(qd, bf16);
  cudaLaunchConfig_t c1 = {};
  c1.gridDim = dim3((r + kLoraJ - 1) / kLoraJ, n_ks, (M + kLoraT - 1) / kLoraT);
  c1.blockDim = dim3(kLoraThreads);
  c1.stream = st;
  c1.attrs = attr;
  c1.numAttrs = pdl ? 1 : 0;
  cudaLaunchConfig_t c2 = c1;
  c2.gridDim = dim3((d + 127) / 128, (M + 7) / 8);
  c2.blockDim = dim3(128);
  cudaError_t e;
  if (bf16 && hilo) {
    using T = __nv_bfloat16;
    e = cudaLaunchKernelEx(&c1, lora_down_kernel<T, true>, static_cast<const T*>(A), static_cast<const T*>(att),
                           static_cast<size_t>(qd), zp, M, qd, r, LoraFinal{});
    if (e == cudaSuccess)
      e = cudaLaunchKernelEx(&c2, lora_up_kernel<T, true>, static_cast<const T*>(B), static_cast<const float*>(zp),
                             h, M, d, r, n_ks, scale, m, causal_rows, causal_seq);
  } else if (bf16) {
    using T = __nv_bfloat16;
    e = cudaLaunchKernelEx(&c1, lora_down_kernel<T, false>, static_cast<const T*>(A), static_cast<const T*>(att),
                           static_cast<size_t>(qd), zp, M, qd, r, LoraFinal{});
    if (e == cudaSuccess)
      e = cudaLaunchKernelEx(&c2, lora_up_kernel<T, false>, static_cast<const T*>(B), static_cast<const float*>(zp),
                             h, M, d, r, n_ks, scale, m, causal_rows, causal_seq);
  } else {
    e = cudaLaunchKernelEx(&c1, lora_down_kernel<float, false>, static_cast<const float*>(A),
                           static_cast<const float*>(att), static_cast<size_t>(qd), zp, M, qd, r, LoraFinal{});
    if (e == cudaSuccess)
      e = cudaLaunchKernelEx(&c2, lora_up_kernel<float, false>, static_cast<const float*>(B),
                             static_cast<const float*>(zp), h, M, d, r, n_ks, scale, m, causal_rows,
                             causal_seq);
  }
  return e;
}

cudaError_t launch_lora_z(cudaStream_t st, const void* A, const void* att, size_t att_ld, float* zp,
                          int* cnt, void* zout, size_t ld, int M, int qd, int r, float scale, int m,
                          int causal_rows, const int* causal_seq, bool pdl) {
  if (r < 8 || r > 256 || r % 8 || M < 1 || !cnt || !zout) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c1 = {};
  c1.gridDim = dim3((r + kLoraJ - 1) / kLoraJ, lora_n_ks(qd, true), (M + kLoraT - 1) / kLoraT);
  c1.blockDim = dim3(kLoraThreads);
  c1.stream = st;
  c1.attrs = attr;
  c1.numAttrs = pdl ? 1 : 0;
  using T = __nv_bfloat16;
  const LoraFinal fin{cnt, static_cast<T*>(zout), ld, scale, m, causal_rows, causal_seq};
  return cudaLaunchKernelEx(&c1, lora_down_kernel<T, true>, static_cast<const T*>(A), static_cast<const T*>(att),
                            att_ld, zp, M, qd, r, fin);
}

// -------------------------------------------------------------------------------- repack --
// dst <- src[row_map[r], c] * gamma[c]  (gamma: RMSNorm gain folded into the projection that
// follows the norm).  Row-major dst[r, c], or, with `tiled`, the streaming layout of the
// tensor-core GEMM: 128-row x 64-column blocks stored contiguously (16 KB of bf16 each), block
// (row tile rt, k tile kt) at element offset (rt * KT + kt) * 8192, rows past n_rows zero.
// Each block holds the byte image the MMA reads from shared memory: row r of the block is 128
// bytes at r * 128 whose eight 16-byte pieces are permuted by the 128-byte swizzle (piece p of
// the row stored at position p ^ (r & 7)), so one plain bulk copy of consecutive blocks into a
// 1024-byte-aligned buffer gives the K-major swizzled operand.
template <typename T>
__global__ void repack_kernel(T* __restrict__ dst, const T* __restrict__ src,
                              const int* __restrict__ row_map, int n_rows, int K,
                              const T* __restrict__ gamma, int tiled) {
  const int row_tiles = (n_rows + kTileRows - 1) / kTileRows;
  const int KT = K / kTileK;
  const size_t total = tiled ? static_cast<size_t>(row_tiles) * kTileRows * K
                             : static_cast<size_t>(n_rows) * K;
  for (size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
    int r, c;
    if (tiled) {
      const size_t blk = idx / (kTileRows * kTileK);
      const int in = static_cast<int>(idx - blk * (kTileRows * kTileK));
      const int rt = static_cast<int>(blk / KT);
      const int kt = static_cast<int>(blk - static_cast<size_t>(rt) * KT);
      // position `in` of the block: row in / 64, 16-byte piece (in % 64) / 8 holds the source
      // piece ((in % 64) / 8) ^ (row & 7)
      const int rr = in / kTileK, pc = ((in % kTileK) >> 3) ^ (rr & 7);
      r = rt * kTileRows + rr;
      c = kt * kTileK + pc * 8 + (in & 7);
    } else {
      r = static_cast<int>(idx / K);
      c = static_cast<int>(idx - static_cast<size_t>(r) * K);
    }
    float v = 0.f;
    if (r < n_rows) {
      const int sr = row_map ? row_map[r] : r;
      v = to_f32<T>(src[static_cast<size_t>(sr) * K + c]);
      if (gamma) v *= to_f32<T>(gamma[c]);
    }
    dst[idx] = from_f32<T>(v);
  }
}

cudaError_t launch_repack(cudaStream_t st, void* dst, const void* src, const int* row_map,
                          int n_rows, int K, const void* gamma, bool bf16, bool tiled) {
  const int threads = 256;
  const size_t total = static_cast<size_t>((n_rows + kTileRows - 1) / kTileRows) * kTileRows * K;
  const int blocks = static_cast<int>(std::min<size_t>((total + threads - 1) / threads, 65536));
  if (bf16)
    repack_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
        static_cast<__nv_bfloat16*>(dst), static_cast<const __nv_bfloat16*>(src), row_map, n_rows,
        K, static_cast<const __nv_bfloat16*>(gamma), tiled ? 1 : 0);
  else
    repack_kernel<float><<<blocks, threads, 0, st>>>(static_cast<float*>(dst),
                                                     static_cast<const float*>(src), row_map,
                                                     n_rows, K, static_cast<const float*>(gamma),
                                                     tiled ? 1 : 0);
  return cudaGetLastError();
}

// ----------------------------------------------------------- stand-alone LM-head helpers --
// ssq[t * M + row] = sum over columns 128t..128t+127 of h[row, c]^2 (fp32), one warp per tile.
__global__ void __launch_bounds__(256) rms_stats_kernel(const __nv_bfloat16* __restrict__ h, int M,
                                                        int d, float* __restrict__ ssq, int* err) {
  const int row = blockIdx.x;
  if (row == 0 && threadIdx.x == 0) *err = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* hr = h + static_cast<size_t>(row) * d;
  for (int t = warp; t < d / kTileRows; t += 8) {
    float sq = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float v = __bfloat162float(hr[t * kTileRows + lane * 4 + q]);
      sq += v * v;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) ssq[static_cast<size_t>(t) * M + row] = sq;
  }
}

cudaError_t launch_rms_stats(cudaStream_t st, const void* h, int M, int d, float* ssq, int* err) {
  rms_stats_kernel<<<M, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h), M, d, ssq, err);
  return cudaGetLastError();
}

// One warp per token: max over vocab tiles (lowest id on ties), then sum_t se_t exp(mx_t - max);
// the confidence is its inverse (largest softmax probability).
__global__ void __launch_bounds__(256) lm_combine_kernel(const LmPart* __restrict__ part, int M,
                                                         int tiles, int* __restrict__ argmax,
                                                         float* __restrict__ conf, const int* err) {
  const int tok = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= M) return;
  if (*err) {   // a wait of the LM-head GEMM ran out: its partials are incomplete
    if (lane == 0) {
      argmax[tok] = -1;
      conf[tok] = 0.f;
    }
    return;
  }
  const LmPart* row = part + static_cast<size_t>(tok) * tiles;
  float mx = -INFINITY;
  int ix = INT_MAX;
  for (int t = lane; t < tiles; t += 32) {
    const LmPart p = row[t];
    if (p.mx > mx || (p.mx == mx && p.idx < ix)) {
      mx = p.mx;
      ix = p.idx;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mx, off);
    const int oi = __shfl_xor_sync(0xffffffffu, ix, off);
    if (om > mx || (om == mx && oi < ix)) {
      mx = om;
      ix = oi;
    }
  }
  float se = 0.f;
  for (int t = lane; t < tiles; t += 32) se += row[t].se * expf(row[t].mx - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) se += __shfl_xor_sync(0xffffffffu, se, off);
  if (lane == 0) {
    argmax[tok] = ix;
    conf[tok] = 1.0f / se;
  }
}

cudaError_t launch_lm_combine(cudaStream_t st, const LmPart* part, int M, int tiles, int* argmax,
                              float* conf, const int* err) {
  lm_combine_kernel<<<(M + 7) / 8, 256, 0, st>>>(part, M, tiles, argmax, conf, err);
  return cudaGetLastError();
}

__global__ void fill_i32_kernel(int* p, int value, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = value;
}

cudaError_t launch_fill_i32(cudaStream_t st, int* p, int value, int n) {
  if (n <= 0) return cudaSuccess;
  fill_i32_kernel<<<(n + 255) / 256, 256, 0, st>>>(p, value, n);
  return cudaGetLastError();
}

}  // namespace nld
