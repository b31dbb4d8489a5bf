// Projection GEMM on the 5th-generation tensor cores (tcgen05), Y^T = W * X^T.
//
// Swap-AB: the weight matrix W [n_rows, K] is the MMA's M=128 operand and the few token rows
// X [M, K] are its N operand (N = 16..256), so a decode forward with 32 or 33 tokens per
// sequence streams every weight byte exactly once.
//
// Split-K across a thread-block cluster: the `split` CTAs of a cluster share each output tile
// (128 weight rows x NT tokens); rank r streams the r-th K slice of the tile into its own
// tensor-memory accumulator.  The partials meet in shared memory: every rank copies its
// accumulator into a staging buffer, tells the other ranks with a remote mbarrier arrive, and
// then reduces one slice of the tile's token columns by reading all ranks' staging buffers over
// distributed shared memory (in rank order, so sums do not depend on timing) and runs the fused
// epilogue on that slice.  Clusters are persistent: cluster c handles tiles c, c+C, ...  With
// split = 1 (large token counts) a tile is finished straight from tensor memory.
//
// Warp roles (192 threads): warp 0 issues TMA loads (W with an evict-first L2 hint), warp 1
// owns tensor memory and issues tcgen05.mma from one thread, warps 2..5 run the epilogue.  A
// `stages`-deep ring of shared-memory stages (16 KB of W + NT*128 B of X each) is guarded by
// full/empty mbarriers; two TMEM accumulators and two staging buffers let the epilogue of one
// tile overlap the MMAs of the next.  Under programmatic dependent launch the first `stages`
// weight tiles are requested before waiting for the previous kernel; activations are read only
// after the wait.  Every wait is bounded (timeout -> device error word, orderly exit).
#include <algorithm>

#include "common.cuh"
#include "epilogue.cuh"

namespace nld {

namespace {

constexpr int kStageW = kTileRows * kTileK * 2;   // 16 KB of bf16 weights per stage
constexpr int kMaxStages = 8;
constexpr int kMaxSplit = 8;

struct GemmTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t sfull[2];    // staging buffer b holds every rank's partial (count: split)
  uint64_t sempty[2];   // every rank has finished reading staging buffer b (count: split)
  uint32_t tmem_base;
  volatile int abort_flag;
  volatile int epi_abort;
  int pad;
  float inv[kMaxNT];
  int pos[kMaxNT];
  int pg[kMaxNT];
  float red_f[96];
  int red_i[96];
};

// Phase timestamps of one CTA (profiling hook): slot i of trace[cta * 16 + i].
NLD_DEV void trace_mark(const GemmShape& s, int slot) {
  if (s.trace) s.trace[blockIdx.x * 16 + slot] = globaltimer_ns();
}

NLD_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, GemmTail* tail,
                           int* err) {
  if (tail->abort_flag) return false;
  if (mbar_wait(bar, parity, timeout_ns)) return true;
  tail->abort_flag = 1;
  set_err(err, NLD_DEVERR_TIMEOUT);
  return false;
}

// Epilogue-side wait: a thread whose wait ran out raises epi_abort before the barrier and every
// epilogue thread reads it after the barrier, so they leave the tile loop together.
NLD_DEV bool epi_wait(uint64_t* bar, uint32_t parity, bool cluster_acquire, uint64_t timeout_ns,
                      GemmTail* tail, int* err) {
  const bool ok = cluster_acquire ? mbar_wait_cluster(bar, parity, timeout_ns)
                                  : mbar_wait(bar, parity, timeout_ns);
  if (!ok) {
    tail->epi_abort = 1;
    set_err(err, NLD_DEVERR_TIMEOUT);
  }
  named_bar_sync(1, 128);
  return tail->epi_abort == 0;
}

}  // namespace

template <int EPI, typename T>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmWn, const GemmShape s, const EpiArgs e_in,
                   const uint64_t timeout_ns) {
  EpiArgs e = e_in;
  e.kind = EPI;   // compile-time epilogue: each instantiation holds one kind's code
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = s.stages;
  const int xbytes = s.NT * 128;
  const int split = s.split;
  uint8_t* sW = smem;
  uint8_t* sX = smem + S * kStageW;
  float* staging = reinterpret_cast<float*>(sX + S * xbytes);          // [2][NT][128] if split>1
  const int stg_floats = (split > 1) ? s.NT * kTileRows : 0;
  GemmTail* tail = reinterpret_cast<GemmTail*>(staging + 2 * stg_floats);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (split > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  const int cl = blockIdx.x / split;
  const int C = gridDim.x / split;
  const int tiles = s.row_tiles * s.tok_tiles;
  const int k_lo = rank * s.ks;
  const int k_hi = min(s.KT, k_lo + s.ks);
  if (threadIdx.x == 0) trace_mark(s, 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&tail->full[i], 1);
      mbar_init(&tail->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tail->tfull[i], 1);
      mbar_init(&tail->tempty[i], 128);
      mbar_init(&tail->sfull[i], split);
      mbar_init(&tail->sempty[i], split);
    }
    tail->abort_flag = 0;
    tail->epi_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, s.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (split > 1) cluster_sync();   // every rank's barriers exist before any remote arrive
  const uint32_t tmem = tail->tmem_base;
  const uint32_t buf_cols = s.tmem_cols / 2;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------- TMA producer --
      const uint64_t pol = l2_policy_evict_first();
      int pre_k[kMaxStages], pre_tt[kMaxStages];
      int npre = 0;
      bool waited = false;
      int it = 0;
      bool ok = true;
      for (int t = cl; ok && t < tiles; t += C) {
        const int r = t / s.tok_tiles;
        const int tt = t - r * s.tok_tiles;
        for (int kt = k_lo; kt < k_hi; ++kt, ++it) {
          const int stage = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          if (!wait_or_abort(&tail->empty[stage], ph ^ 1u, timeout_ns, tail, e.err)) {
            ok = false;
            break;
          }
          if (it == 0) trace_mark(s, 2);
          mbar_arrive_expect_tx(&tail->full[stage], kStageW + xbytes);
          tma_load_2d_hint(sW + stage * kStageW, &tmW, &tail->full[stage], kt * kTileK,
                           r * kTileRows, pol);
          if (waited) {
            tma_load_2d(sX + stage * xbytes, &tmX, &tail->full[stage], kt * kTileK, tt * s.NT);
          } else {
            pre_k[npre] = kt;
            pre_tt[npre] = tt;
            if (++npre == S) {
              pdl_wait();
              waited = true;
              for (int i = 0; i < npre; ++i)
                tma_load_2d(sX + i * xbytes, &tmX, &tail->full[i], pre_k[i] * kTileK,
                            pre_tt[i] * s.NT);
            }
          }
        }
      }
      if (!waited) {
        pdl_wait();
        for (int i = 0; i < npre; ++i)
          tma_load_2d(sX + i * xbytes, &tmX, &tail->full[i], pre_k[i] * kTileK, pre_tt[i] * s.NT);
      }
      trace_mark(s, 3);
      if (ok && s.next_valid && blockIdx.x < s.next_clusters * s.next_split) {
        // warm L2 (and address translation) for this CTA index's first boxes of the next GEMM
        const int nrank = blockIdx.x % s.next_split;
        const int ncl = blockIdx.x / s.next_split;
        if (ncl < s.next_tiles) {
          const int nr = ncl / s.next_tok_tiles;
          const int lo = nrank * s.next_ks;
          const int hi = min(s.next_KT, min(lo + s.next_ks, lo + s.next_boxes));
          for (int kt = lo; kt < hi; ++kt) tma_prefetch_l2_2d(&tmWn, kt * kTileK, nr * kTileRows);
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA can exit
        const int first = it - S > 0 ? it - S : 0;
        for (int j = first; j < it; ++j)
          mbar_wait(&tail->full[j % S], static_cast<uint32_t>(j / S) & 1u, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer --
      const uint32_t idesc = idesc_bf16_f32(kTileRows, s.NT);
      int it = 0, i = 0;
      bool ok = true;
      for (int t = cl; ok && t < tiles; t += C, ++i) {
        const int tb = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        if (!wait_or_abort(&tail->tempty[tb], (use & 1u) ^ 1u, timeout_ns, tail, e.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + tb * buf_cols;
        for (int kt = k_lo; kt < k_hi; ++kt, ++it) {
          const int stage = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          if (!wait_or_abort(&tail->full[stage], ph, timeout_ns, tail, e.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (it == 0) trace_mark(s, 4);
          const uint64_t da = sdesc_k_sw128(smem_u32(sW + stage * kStageW));
          const uint64_t db = sdesc_k_sw128(smem_u32(sX + stage * xbytes));
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)
            tc_mma_f16(d, da + 2 * kk, db + 2 * kk, idesc, (kt > k_lo || kk > 0) ? 1u : 0u);
          tc_commit(&tail->empty[stage]);
        }
        if (!ok) break;
        tc_commit(&tail->tfull[tb]);
        trace_mark(s, 5 + (i < 2 ? i : 1));
      }
    }
    __syncwarp();
    // every epilogue read of tensor memory is done once the epilogue warps reach barrier 2
    named_bar_sync(2, 160);
    tc_fence_after();
    tmem_dealloc(tmem, s.tmem_cols);
  } else {
    // -------------------------------------------------------------------- epilogue --
    pdl_wait();
    const int et = threadIdx.x - 64;
    const int ew = warp & 3;              // TMEM lane quarter this warp may read
    const int row_in_tile = ew * 32 + lane;
    const bool need_norm = (EPI != EPI_RESID);
    uint32_t stg_peer[kMaxSplit];
    if (split > 1) {
#pragma unroll
      for (int q = 0; q < kMaxSplit; ++q)
        stg_peer[q] = dsmem_addr(smem_u32(staging), static_cast<uint32_t>(q < split ? q : 0));
    }
    int i = 0;
    for (int t = cl; t < tiles; t += C, ++i) {
      const int r = t / s.tok_tiles;
      const int tt = t - r * s.tok_tiles;
      const int tok0 = tt * s.NT;
      const int nvalid = min(s.NT, e.M - tok0);
      const int nchunks = (nvalid + 15) >> 4;
      const int tb = i & 1;
      const uint32_t use = static_cast<uint32_t>(i >> 1);
      named_bar_sync(1, 128);
      compute_tile_meta(e, tok0, s.NT, need_norm, tail->inv, tail->pos, tail->pg, et, 128);
      if (!epi_wait(&tail->tfull[tb], use & 1u, false, timeout_ns, tail, e.err)) break;
      tc_fence_after();
      if (et == 0) trace_mark(s, 7 + (i < 2 ? i : 1));
      const uint32_t tbase = tmem + (static_cast<uint32_t>(ew * 32) << 16) + tb * buf_cols;
      if (split == 1) {
        for (int c = 0; c < nchunks; ++c) {
          float v[16];
          tmem_ld16(tbase + c * 16, v);
          epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + c * 16, tail->inv, tail->pos, tail->pg,
                       c * 16, v, tail->red_f, tail->red_i);
        }
        tc_fence_before();
        mbar_arrive(&tail->tempty[tb]);
      } else {
        // 1. this rank's partial -> staging buffer b, once every rank has read its last use
        const int b = i & 1;
        if (!epi_wait(&tail->sempty[b], (use & 1u) ^ 1u, true, timeout_ns, tail, e.err)) break;
        float* stg = staging + b * stg_floats;
        for (int c = 0; c < nchunks; ++c) {
          float v[16];
          tmem_ld16(tbase + c * 16, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) stg[(c * 16 + j) * kTileRows + row_in_tile] = v[j];
        }
        tc_fence_before();
        mbar_arrive(&tail->tempty[tb]);
        named_bar_sync(1, 128);
        if (et == 0)
          for (int q = 0; q < split; ++q)
            mbar_arrive_remote(dsmem_addr(smem_u32(&tail->sfull[b]), static_cast<uint32_t>(q)));
        // 2. every rank's partial is staged: reduce this rank's column slice over DSMEM
        if (!epi_wait(&tail->sfull[b], use & 1u, true, timeout_ns, tail, e.err)) break;
        if (et == 0) trace_mark(s, 12);
        const int per = (nchunks + split - 1) / split;
        const int c_lo = rank * per, c_hi = min(nchunks, c_lo + per);
        const uint32_t off0 = static_cast<uint32_t>(b * stg_floats) * 4u;
        for (int c = c_lo; c < c_hi; ++c) {
          float part[kMaxSplit][16];
          const uint32_t cofs = off0 + static_cast<uint32_t>((c * 16) * kTileRows + row_in_tile) * 4u;
#pragma unroll
          for (int q = 0; q < kMaxSplit; ++q) {
            if (q < split) {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                part[q][j] = ld_dsmem_f32(stg_peer[q] + cofs + static_cast<uint32_t>(j * kTileRows * 4));
            }
          }
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < kMaxSplit; ++q)
              if (q < split) acc += part[q][j];
            v[j] = acc;
          }
          epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + c * 16, tail->inv, tail->pos, tail->pg,
                       c * 16, v, tail->red_f, tail->red_i);
        }
        // 3. this rank is done reading every rank's staging buffer b
        named_bar_sync(1, 128);
        if (et == 0)
          for (int q = 0; q < split; ++q)
            mbar_arrive_remote(dsmem_addr(smem_u32(&tail->sempty[b]), static_cast<uint32_t>(q)));
      }
      if (et == 0) trace_mark(s, 9 + (i < 2 ? i : 1));
    }
    tc_fence_before();
    named_bar_sync(2, 160);
    if (et == 0) trace_mark(s, 15);
  }
  // peers may still read this CTA's staging buffers or arrive on its barriers
  if (split > 1) cluster_sync();
  if (threadIdx.x == 0) trace_mark(s, 11);
}

size_t gemm_tc_smem_bytes(const GemmShape& s) {
  const size_t stg = (s.split > 1) ? 2ull * s.NT * kTileRows * sizeof(float) : 0;
  return 1024 + static_cast<size_t>(s.stages) * (kStageW + s.NT * 128) + stg + sizeof(GemmTail);
}

template <int EPI>
static cudaError_t set_smem_limit(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, gemm_tc_kernel<EPI, __nv_bfloat16>);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(gemm_tc_kernel<EPI, __nv_bfloat16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - static_cast<int>(fa.sharedSizeBytes));
}

cudaError_t gemm_tc_init_attributes() {
  int dev = 0, optin = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  if ((e = set_smem_limit<EPI_QKV>(optin)) != cudaSuccess) return e;
  if ((e = set_smem_limit<EPI_RESID>(optin)) != cudaSuccess) return e;
  if ((e = set_smem_limit<EPI_SWIGLU>(optin)) != cudaSuccess) return e;
  if ((e = set_smem_limit<EPI_LMHEAD>(optin)) != cudaSuccess) return e;
  return set_smem_limit<EPI_LOGITS>(optin);
}

// Clusters of `split` CTAs (one CTA per SM at `smem` bytes) that can be resident at once.
int gemm_tc_max_clusters(int split, size_t smem, int sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(split * (sms / split));
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<EPI_QKV, __nv_bfloat16>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return sms / split;
  }
  return n > 0 ? std::min(n, sms / split) : sms / split;
}

cudaError_t launch_gemm_tc(cudaStream_t st, const CUtensorMap* tmW, const CUtensorMap* tmX,
                           const GemmShape& s, const EpiArgs& e, uint64_t timeout_ns, bool pdl,
                           const CUtensorMap* tmW_next) {
  const CUtensorMap* wn = tmW_next ? tmW_next : tmW;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.G);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = gemm_tc_smem_bytes(s);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = s.split;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  switch (e.kind) {
    case EPI_QKV:
      return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_QKV, __nv_bfloat16>, *tmW, *tmX, *wn, s, e,
                                timeout_ns);
    case EPI_RESID:
      return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_RESID, __nv_bfloat16>, *tmW, *tmX, *wn, s, e,
                                timeout_ns);
    case EPI_SWIGLU:
      return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_SWIGLU, __nv_bfloat16>, *tmW, *tmX, *wn, s, e,
                                timeout_ns);
    case EPI_LMHEAD:
      return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_LMHEAD, __nv_bfloat16>, *tmW, *tmX, *wn, s, e,
                                timeout_ns);
    default:
      return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI_LOGITS, __nv_bfloat16>, *tmW, *tmX, *wn, s, e,
                                timeout_ns);
  }
}

}  // namespace nld
