// Small-M projection GEMM on the 5th-generation tensor cores (tcgen05), Y^T = W * X^T.
//
// Swap-AB: the weight matrix W [n_rows, K] is the MMA's M=128 operand and the few token rows
// X [M, K] are its N operand (N = 16..256), so a decode forward with 32 or 33 tokens per
// sequence streams every weight byte exactly once.  Work is split stream-K: the k-iterations
// of all (row tile, token tile) pairs are laid end to end and cut into `G` equal contiguous
// ranges, one per CTA (G <= number of SMs, one CTA per SM), so every SM streams the same
// number of weight bytes.  A tile whose k-range falls inside one CTA is finished from tensor
// memory; a tile cut by a range boundary is finished by whichever of its contributors
// arrives last (atomic counter), which sums the fp32 partials in a fixed order, so results
// do not depend on timing.
//
// Warp roles (192 threads): warp 0 issues TMA loads (W with an evict-first L2 hint), warp 1
// allocates tensor memory and issues tcgen05.mma from one thread, warps 2..5 run the
// epilogue (TMEM -> registers -> fused epilogue).  A `stages`-deep ring of shared-memory
// stages (16 KB of W + NT*128 B of X each) is guarded by full/empty mbarriers; two TMEM
// accumulators let the epilogue of one tile overlap the MMAs of the next.  Under programmatic
// dependent launch the first `stages` weight tiles are requested before waiting for the
// previous kernel; activations are read only after the wait.
#include "common.cuh"
#include "epilogue.cuh"

namespace nld {

namespace {

constexpr int kStageW = kTileRows * kTileK * 2;   // 16 KB of bf16 weights per stage
constexpr int kMaxStages = 8;

struct GemmTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  volatile int abort_flag;
  volatile int epi_abort;
  int last_flag;
  float inv[kMaxNT];
  float red_f[96];
  int red_i[96];
};

struct Seg {
  int tile, k0, k1;
};

NLD_DEV bool next_seg(long long& t, long long t_end, int KT, Seg& s) {
  if (t >= t_end) return false;
  s.tile = static_cast<int>(t / KT);
  s.k0 = static_cast<int>(t - static_cast<long long>(s.tile) * KT);
  const long long rem = t_end - t;
  s.k1 = static_cast<int>(rem < KT - s.k0 ? s.k0 + rem : KT);
  t += s.k1 - s.k0;
  return true;
}

NLD_DEV long long range_begin(int c, long long T, int G) {
  return static_cast<long long>(c) * T / G;
}
// CTA whose range holds k-iteration t: max{c : floor(c*T/G) <= t}.
NLD_DEV int owner_of(long long t, long long T, int G) {
  return static_cast<int>(((t + 1) * G + T - 1) / T) - 1;
}

NLD_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, GemmTail* tail,
                           int* err) {
  if (tail->abort_flag) return false;
  if (mbar_wait(bar, parity, timeout_ns)) return true;
  tail->abort_flag = 1;
  set_err(err, NLD_DEVERR_TIMEOUT);
  return false;
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const GemmShape s, const EpiArgs e, float* __restrict__ ws,
                   int* __restrict__ counters, const uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = s.stages;
  const int xbytes = s.NT * 128;
  uint8_t* sW = smem;
  uint8_t* sX = smem + S * kStageW;
  GemmTail* tail = reinterpret_cast<GemmTail*>(sX + S * xbytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long long t_begin = range_begin(cta, s.T, s.G);
  const long long t_end = range_begin(cta + 1, s.T, s.G);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&tail->full[i], 1);
      mbar_init(&tail->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tail->tfull[i], 1);
      mbar_init(&tail->tempty[i], 128);
    }
    tail->abort_flag = 0;
    tail->epi_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, s.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
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
      long long t = t_begin;
      int it = 0;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(t, t_end, s.KT, sg)) {
        const int r = sg.tile / s.tok_tiles;
        const int tt = sg.tile - r * s.tok_tiles;
        for (int kt = sg.k0; kt < sg.k1; ++kt, ++it) {
          const int stage = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          if (!wait_or_abort(&tail->empty[stage], ph ^ 1u, timeout_ns, tail, e.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], kStageW + xbytes);
          tma_load_2d_hint(sW + stage * kStageW, &tmW, &tail->full[stage], kt * kTileK,
                           r * kTileRows, pol);
          if (waited) {
            tma_load_2d(sX + stage * xbytes, &tmX, &tail->full[stage], kt * kTileK, tt * s.NT);
          } else {
            pre_k[npre] = kt;
            pre_tt[npre] = tt;
            ++npre;
            if (npre == S) {
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
      if (!ok) {
        // drain: let every load already issued land before the CTA can exit
        const int first = it - S > 0 ? it - S : 0;
        for (int j = first; j < it; ++j)
          mbar_wait(&tail->full[j % S], static_cast<uint32_t>(j / S) & 1u, timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer --
      const uint32_t idesc = idesc_bf16_f32(kTileRows, s.NT);
      long long t = t_begin;
      int it = 0, seg = 0;
      Seg sg;
      bool ok = true;
      while (ok && next_seg(t, t_end, s.KT, sg)) {
        const int b = seg & 1;
        const uint32_t use = static_cast<uint32_t>(seg >> 1);
        if (!wait_or_abort(&tail->tempty[b], (use & 1u) ^ 1u, timeout_ns, tail, e.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * buf_cols;
        for (int kt = sg.k0; kt < sg.k1; ++kt, ++it) {
          const int stage = it % S;
          const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
          if (!wait_or_abort(&tail->full[stage], ph, timeout_ns, tail, e.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = sdesc_k_sw128(smem_u32(sW + stage * kStageW));
          const uint64_t db = sdesc_k_sw128(smem_u32(sX + stage * xbytes));
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)
            tc_mma_f16(d, da + 2 * kk, db + 2 * kk, idesc, (kt > sg.k0 || kk > 0) ? 1u : 0u);
          tc_commit(&tail->empty[stage]);
        }
        if (!ok) break;
        tc_commit(&tail->tfull[b]);
        ++seg;
      }
    }
  } else {
    // -------------------------------------------------------------------- epilogue --
    pdl_wait();
    const int et = threadIdx.x - 64;
    const int ew = warp & 3;              // TMEM lane quarter this warp may read
    const int row_in_tile = ew * 32 + lane;
    const bool need_norm = (e.kind != EPI_RESID);
    const int first_tile_mine = static_cast<int>(t_begin / s.KT);
    long long t = t_begin;
    int seg = 0;
    Seg sg;
    while (next_seg(t, t_end, s.KT, sg)) {
      const int b = seg & 1;
      const uint32_t use = static_cast<uint32_t>(seg >> 1);
      const int r = sg.tile / s.tok_tiles;
      const int tt = sg.tile - r * s.tok_tiles;
      const int tok0 = tt * s.NT;
      const int nvalid = min(s.NT, e.M - tok0);
      const int nchunks = (nvalid + 15) >> 4;
      named_bar_sync(1, 128);
      if (need_norm) compute_inv_rms(e, tok0, s.NT, tail->inv, et, 128);
      named_bar_sync(1, 128);
      // Uniform exit: a thread whose wait ran out raises epi_abort before the barrier and
      // every epilogue thread reads it after the barrier, so none is left at a later one.
      if (!mbar_wait(&tail->tfull[b], use & 1u, timeout_ns)) {
        tail->epi_abort = 1;
        set_err(e.err, NLD_DEVERR_TIMEOUT);
      }
      named_bar_sync(1, 128);
      if (tail->epi_abort) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(ew * 32) << 16) + b * buf_cols;
      const bool whole = (sg.k0 == 0 && sg.k1 == s.KT);
      if (whole) {
        for (int c = 0; c < nchunks; ++c) {
          float v[16];
          tmem_ld16(tbase + c * 16, v);
          epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + c * 16, tail->inv, c * 16, v,
                       tail->red_f, tail->red_i);
        }
        tc_fence_before();
        mbar_arrive(&tail->tempty[b]);
      } else {
        const int slot = (sg.tile == first_tile_mine) ? 0 : 1;
        float* dst = ws + (static_cast<size_t>(cta) * 2 + slot) * s.ws_slot;
        for (int c = 0; c < nchunks; ++c) {
          float v[16];
          tmem_ld16(tbase + c * 16, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) dst[(c * 16 + j) * kTileRows + row_in_tile] = v[j];
        }
        tc_fence_before();
        mbar_arrive(&tail->tempty[b]);
        __threadfence();
        named_bar_sync(1, 128);
        const long long kfirst = static_cast<long long>(sg.tile) * s.KT;
        const int c_first = owner_of(kfirst, s.T, s.G);
        const int c_last = owner_of(kfirst + s.KT - 1, s.T, s.G);
        if (et == 0) {
          const int old = atomicAdd(&counters[sg.tile], 1);
          const int last = (old == c_last - c_first) ? 1 : 0;
          if (last) counters[sg.tile] = 0;
          tail->last_flag = last;
        }
        named_bar_sync(1, 128);
        if (tail->last_flag) {
          __threadfence();
          for (int c = 0; c < nchunks; ++c) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            for (int cc = c_first; cc <= c_last; ++cc) {
              const int first_cc = static_cast<int>(range_begin(cc, s.T, s.G) / s.KT);
              const int sl = (sg.tile == first_cc) ? 0 : 1;
              const float* src = ws + (static_cast<size_t>(cc) * 2 + sl) * s.ws_slot;
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] += __ldcg(src + (c * 16 + j) * kTileRows + row_in_tile);
            }
            epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + c * 16, tail->inv, c * 16, v,
                         tail->red_f, tail->red_i);
          }
        }
      }
      ++seg;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, s.tmem_cols);
  }
}

cudaError_t gemm_tc_init_attributes() {
  int dev = 0, optin = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, gemm_tc_kernel<__nv_bfloat16>)) != cudaSuccess) return e;
  return cudaFuncSetAttribute(gemm_tc_kernel<__nv_bfloat16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - static_cast<int>(fa.sharedSizeBytes));
}

size_t gemm_tc_smem_bytes(const GemmShape& s) {
  return 1024 + static_cast<size_t>(s.stages) * (kStageW + s.NT * 128) + sizeof(GemmTail);
}

cudaError_t launch_gemm_tc(cudaStream_t st, const CUtensorMap* tmW, const CUtensorMap* tmX,
                           const GemmShape& s, const EpiArgs& e, float* ws, int* counters,
                           uint64_t timeout_ns, bool pdl) {
  const size_t smem = gemm_tc_smem_bytes(s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(s.G);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<__nv_bfloat16>, *tmW, *tmX, s, e, ws, counters,
                            timeout_ns);
}

}  // namespace nld
