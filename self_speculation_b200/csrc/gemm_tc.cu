// Projection GEMMs on the 5th-generation tensor cores (tcgen05), Y^T = W * X^T, run as a
// persistent chain: one launch executes up to four projections back to back (for a decode
// layer: O-proj, gate/up, down, and the next layer's QKV, or for the last layer the final
// norm + LM head).
//
// Swap-AB: the weight matrix W [n_rows, K] is the MMA's M=128 operand and the few token rows
// X [M, K] are its N operand (N = 16..256), so a decode forward streams every weight byte once.
// Activations are fp32 values held as two bf16 rows each (hi = bf16(x), lo = bf16(x - hi),
// interleaved: row 2t, 2t+1 for token t), so one MMA of N = 2 x tokens multiplies both halves by
// the same weights and the epilogue adds column pairs: the product has the precision of fp32
// operands against bf16 weights (the stand-alone LM head over caller bf16 rows uses N = tokens).
// Weights are stored pre-tiled (128 x 64 blocks, 16 KB contiguous), so each TMA box is one
// contiguous read and a CTA's K range is one contiguous stretch of HBM.  A pipeline stage holds
// two k-tiles (32 KB of weights plus the activation rows), so one producer -> MMA -> producer
// barrier round trip moves 32 KB.
//
// Work split: the CTAs of a cluster (CS of them) share output tiles; in a phase with split s
// (a divisor of CS) each group of s ranks splits the K range of a tile, each rank accumulating
// its slice in tensor memory.  The tile's 16-column chunks are divided among the group; every
// rank sends its partial of each chunk to the chunk's owner with st.async (a one-way write into
// the owner's shared memory, counted by the owner's mbarrier), and the owner sums the partials
// in rank order (sums do not depend on timing) and runs the fused epilogue on them.
//
// Phases: a CTA that finished its part of phase p adds one to a grid-wide arrival counter; the
// next phase's activation loads and epilogue wait until every CTA has arrived.  Its weight
// loads do not wait: the producer keeps the shared-memory ring full with the next phase's
// weights across the transition and, while it waits, prefetches the following boxes into L2,
// so HBM stays busy while the last tiles of a phase finish.
// The first phase waits for the previous kernel the same way (programmatic dependent launch).
//
// Warp roles (320 threads): warp 0 issues TMA loads (W with an evict-first L2 hint), warp 1
// owns tensor memory and issues tcgen05.mma from one thread, warps 2..9 run the epilogue: two
// warps per TMEM lane quarter, alternating 16-column chunks.
// Every wait is bounded (timeout -> device error word, orderly exit).
#include <algorithm>

#include "common.cuh"
#include "epilogue.cuh"

namespace nld {

namespace {

constexpr int kStageW = kTileRows * kTileK * 2;   // 16 KB: one k-tile of bf16 weights
constexpr int kMaxStages = 8;
constexpr int kSlotLd = 16;              // floats per row of a split-K slot (one 16-column chunk)
constexpr int kSlotFloats = kTileRows * kSlotLd;
// Byte offset of 16-byte piece q (0..3) of `row` in a slot: the pieces of a row are permuted by
// (row >> 1) & 3 so that the 16-byte accesses of 8 consecutive rows hit distinct bank groups.
NLD_DEV uint32_t slot_off(int row, int q) {
  return static_cast<uint32_t>(row * kSlotLd * 4 + ((q ^ ((row >> 1) & 3)) << 4));
}
constexpr int kEpiThreads = 256;   // 8 epilogue warps
constexpr int kThreads = 64 + kEpiThreads;

struct GemmTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t rfull;       // the group's partials of this CTA's chunks have arrived (count 1 + tx)
  uint32_t done[kMaxPhases];   // split tiles of phase p whose chunks this CTA has reduced (read
                               // by the group's other ranks before they write its slot area)
  uint32_t tmem_base;
  volatile int abort_flag;
  volatile int epi_abort;
  int pad;
  float red_f[2][80];   // per epilogue half (4 x 16 partials + 16 results)
  int red_i[2][80];
  // the producer's queued activation loads (one thread; in shared memory, the dynamically
  // indexed arrays stay out of local memory, which goes to L2 with the unified L1 given to the
  // ring)
  int q_stage[kMaxStages], q_k[kMaxStages], q_tt[kMaxStages], q_nk[kMaxStages];
  // followed in shared memory by the tile's per-column data: inv[NT], pos[NT], pg[NT], rpos[NT]
};

// Work of one CTA in phase p: its group of s ranks, the group's tiles and this rank's K slice.
struct Work {
  int s, grank, grp, ngrp, tiles, k_lo, k_hi;
};

NLD_DEV Work work_of(const ChainArgs& A, int p, int cl, int rank, int C) {
  const PhaseArgs& P = A.ph[p];
  Work w;
  w.s = P.s;
  const int gpc = A.CS / P.s;
  w.grank = rank % P.s;
  w.grp = cl * gpc + rank / P.s;
  w.ngrp = C * gpc;
  w.tiles = P.row_tiles * P.tok_tiles;
  w.k_lo = w.grank * P.ks;
  w.k_hi = min(P.KT, w.k_lo + P.ks);
  return w;
}

// Transaction bytes of the next split tile after tile t_prev of phase p (t_prev = -1: from the
// start of phase p) in which this CTA owns chunks: every other rank of the group sends it 64
// bytes per row per owned chunk.  0 if there is none.
NLD_DEV uint32_t next_owned_bytes(const ChainArgs& A, int p, int t_prev, int cl, int rank, int C) {
  for (int q = p; q < A.nph; ++q) {
    const PhaseArgs& P = A.ph[q];
    const Work w = work_of(A, q, cl, rank, C);
    if (w.s <= 1) continue;
    for (int t = (q == p && t_prev >= 0) ? t_prev + w.ngrp : w.grp; t < w.tiles; t += w.ngrp) {
      const int tt = t - (t / P.tok_tiles) * P.tok_tiles;
      const int nvalid = min(A.NT, P.e.M - tt * A.NT);
      const int nchunks = (nvalid + 15) >> 4;
      const int per = (nchunks + w.s - 1) / w.s;
      const int n_own = min(nchunks, (w.grank + 1) * per) - w.grank * per;
      if (n_own > 0) return static_cast<uint32_t>((w.s - 1) * n_own * kTileRows * 64);
    }
  }
  return 0;
}

// Phase timestamps of one CTA (profiling hook), trace[cta * 16 + slot]: 0 start, 1 set-up
// done, per phase p: 2+3p first weight load issued, 3+3p epilogue may start (after the phase
// counter), 4+3p epilogue done; 14 last MMA commit, 15 exit.
NLD_DEV void trace_mark(const ChainArgs& A, int slot) {
  if (A.trace) A.trace[blockIdx.x * 16 + slot] = globaltimer_ns();
}
// Per-iteration pipeline stamps of CTA 0 (profiling hook), after the per-CTA slots: kind 0
// stage `it` issued, 1 stage `it` consumed by the MMA, 2 stage `it` freed; kind 3 at 8i + k
// for the epilogue of tile i: k = 0 accumulator ready, 1 partials sent, 2 the group's partials
// received, 3 reduced and written (all threads), 4 done, 5 / 6 thread 0's sums formed / its
// chunk written.
NLD_DEV void trace_iter(const ChainArgs& A, int kind, int it) {
  if (A.trace && blockIdx.x == 0 && it >= 0 && it < 64)
    A.trace[kChainTraceEntries - 4 * 64 + kind * 64 + it] = globaltimer_ns();
}

// The accumulator of chunk c (16 tokens) of a tile.  With hi/lo activations (rows 2t, 2t+1 =
// bf16(x_t), bf16(x_t - bf16(x_t))) columns 2t and 2t+1 hold W x_hi and W x_lo of token t, and
// their sum is W x_t to fp32-operand precision.
NLD_DEV void tmem_ld_chunk(uint32_t tbase, int c, int hilo, float (&v)[16]) {
  if (!hilo) {
    tmem_ld16(tbase + c * 16, v);
    return;
  }
  uint32_t a[16], b[16];
  tmem_ld16_nowait(tbase + c * 32, a);
  tmem_ld16_nowait(tbase + c * 32 + 16, b);
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[j] = __uint_as_float(a[2 * j]) + __uint_as_float(a[2 * j + 1]);
    v[8 + j] = __uint_as_float(b[2 * j]) + __uint_as_float(b[2 * j + 1]);
  }
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
// epilogue thread reads it after the barrier, so they leave together.
NLD_DEV bool epi_wait(uint64_t* bar, uint32_t parity, bool cluster_acquire, uint64_t timeout_ns,
                      GemmTail* tail, int* err) {
  const bool ok = cluster_acquire ? mbar_wait_cluster(bar, parity, timeout_ns)
                                  : mbar_wait(bar, parity, timeout_ns);
  if (!ok) {
    tail->epi_abort = 1;
    set_err(err, NLD_DEVERR_TIMEOUT);
  }
  named_bar_sync(1, kEpiThreads);
  return tail->epi_abort == 0;
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_chain_kernel(const __grid_constant__ ChainArgs A, const uint64_t timeout_ns) {
  // the launch asks for no alignment slack: the dynamic shared memory of a CTA without static
  // shared memory starts 1024-byte aligned, which the 128-byte swizzle of the ring needs; a launch
  // where it does not leaves at once (error word) before any barrier or tensor-memory use
  extern __shared__ uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) set_err(A.ph[0].e.err, NLD_DEVERR_LAUNCH);
    return;
  }
  uint8_t* smem = smem_raw;
  const int S = A.stages;
  const int NT = A.NT;
  const int NN = NT << A.hilo;         // MMA N: activation rows of a token tile (hi/lo pairs)
  const int KPS = A.kps;
  const int xbytes = A.xr * 128;       // one k-tile of activations: xr token rows x 128 B
  const int wst = KPS * kStageW;       // one stage: KPS k-tiles of weights ...
  const int xst = KPS * xbytes;        // ... and of activations
  const int CS = A.CS;
  uint8_t* sW = smem;
  uint8_t* sX = smem + S * wst;
  // split-K slot area (CS > 1): [A.slots][128 rows][kSlotLd] floats; for a split tile of group
  // size s, slot (q' * per + c) holds the partial of this CTA's c-th owned chunk from the q'-th
  // other rank of the group (q' = q for ranks q below this one, q - 1 above); the owner keeps
  // its own partial in registers
  float* slots = reinterpret_cast<float*>(sX + S * xst);
  GemmTail* tail = reinterpret_cast<GemmTail*>(slots + (CS > 1 ? A.slots * kSlotFloats : 0));
  float* const s_inv = reinterpret_cast<float*>(tail + 1);
  int* const s_pos = reinterpret_cast<int*>(s_inv + NT);
  int* const s_pg = s_pos + NT;
  int* const s_rpos = s_pg + NT;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (CS > 1) ? static_cast<int>(cluster_ctarank()) : 0;
  const int cl = blockIdx.x / CS;
  const int C = gridDim.x / CS;
  const unsigned G = gridDim.x;
  int* err = A.ph[0].e.err;
  if (threadIdx.x == 0) trace_mark(A, 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&tail->full[i], 1);
      mbar_init(&tail->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tail->tfull[i], 1);
      mbar_init(&tail->tempty[i], kEpiThreads);
    }
    mbar_init(&tail->rfull, 1);
    for (int p = 0; p < kMaxPhases; ++p) tail->done[p] = 0;
    tail->abort_flag = 0;
    tail->epi_abort = 0;
    fence_mbar_init();
    // the first split tile whose chunks this CTA owns: its transaction count is armed before
    // any rank of the cluster can send (they all pass the cluster barrier below first)
    if (CS > 1) {
      const uint32_t b0 = next_owned_bytes(A, 0, -1, blockIdx.x / CS, static_cast<int>(cluster_ctarank()),
                                           static_cast<int>(gridDim.x) / CS);
      if (b0) mbar_arrive_expect_tx(&tail->rfull, b0);
    }
    for (int p = 0; p < A.nph; ++p) {
      tma_prefetch_desc(&A.ph[p].tmW);
      tma_prefetch_desc(&A.ph[p].tmX);
    }
  }
  __syncwarp();
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, A.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (CS > 1) cluster_sync();   // every rank's barriers exist before any remote arrive
  const uint32_t tmem = tail->tmem_base;
  const uint32_t buf_cols = A.tmem_cols / 2;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------- TMA producer --
      const uint64_t pol = l2_policy_evict_first();
      int* q_stage = tail->q_stage;
      int* q_k = tail->q_k;
      int* q_tt = tail->q_tt;
      int* q_nk = tail->q_nk;
      int it = 0;
      int n_issued = 0;   // stages whose loads were issued
      bool ok = true;
      // L2 run-ahead (A.pf_stages = D > 0, pre-tiled weights): after the load of stage `it` is
      // issued, the weights of stage it + D are prefetched into L2 with one bulk prefetch of their
      // contiguous blocks, so the load of that stage finds them there.  The cursor walks the
      // same (phase, tile, k) order as the loads; divisions only where it enters a phase.
      struct PfCursor {
        int p, t, kt, k_lo, k_hi, ngrp, tiles, tok_tiles, KT;
        const uint8_t* W;
        bool live;
      } pf{};
      auto pf_phase = [&](int q) {
        pf.live = false;
        for (; q < A.nph; ++q) {
          const PhaseArgs& Q = A.ph[q];
          if (Q.w_rowmajor) return;
          const Work wq = work_of(A, q, cl, rank, C);
          if (wq.grp < wq.tiles) {
            pf = {q, wq.grp, wq.k_lo, wq.k_lo, wq.k_hi, wq.ngrp, wq.tiles, Q.tok_tiles, Q.KT,
                  static_cast<const uint8_t*>(Q.W), true};
            return;
          }
        }
      };
      auto pf_step = [&](bool issue) {
        if (!pf.live) return;
        if (issue) {
          const int r = (pf.tok_tiles == 1) ? pf.t : pf.t / pf.tok_tiles;
          bulk_prefetch_l2(pf.W + (static_cast<size_t>(r) * pf.KT + pf.kt) * kStageW,
                           static_cast<uint32_t>(min(KPS, pf.k_hi - pf.kt) * kStageW));
        }
        pf.kt += KPS;
        if (pf.kt >= pf.k_hi) {
          pf.kt = pf.k_lo;
          pf.t += pf.ngrp;
          if (pf.t >= pf.tiles) pf_phase(pf.p + 1);
        }
      };
      if (A.pf_stages > 0) {
        // the first S stages fill the ring at once: the run-ahead starts after them
        pf_phase(0);
        for (int i = 0; i < S; ++i) pf_step(false);
        for (int i = 0; i < A.pf_stages; ++i) pf_step(true);
      }
      for (int p = 0; ok && p < A.nph; ++p) {
        const PhaseArgs& P = A.ph[p];
        const Work w = work_of(A, p, cl, rank, C);
        // activation loads of this phase wait for the previous kernel (p == 0) or for every
        // CTA to finish phase p-1; weight loads run ahead into the free stages meanwhile
        bool ready = false;
        int nq = 0;
        // (tn, ktn): the next weight box this CTA loads after the ring's queued stages; while
        // the phase boundary is waited on, the TMA unit is idle, so it prefetches the following
        // boxes into L2 and HBM keeps streaming through the boundary
        auto become_ready = [&](int tn, int ktn) -> bool {
          if (p == 0) {
            pdl_wait();
          } else {
            const uint64_t t0 = globaltimer_ns();
            int npf = 0;
            while (ld_acquire_gpu(A.bar + (p - 1)) < G) {
              if (npf < A.boundary_pf && tn < w.tiles) {
                const int rn = tn / P.tok_tiles;
                if (P.w_rowmajor)
                  tma_prefetch_l2_2d(&P.tmW, ktn * kTileK, rn * kTileRows);
                else
                  bulk_prefetch_l2(static_cast<const uint8_t*>(P.W) +
                                       (static_cast<size_t>(rn) * P.KT + ktn) * kStageW, kStageW);
                ++npf;
                if (++ktn >= w.k_hi) {
                  tn += w.ngrp;
                  ktn = w.k_lo;
                }
              } else if (globaltimer_ns() - t0 > timeout_ns) {
                tail->abort_flag = 1;
                set_err(err, NLD_DEVERR_TIMEOUT);
                return false;
              }
            }
            fence_proxy_async_global();
          }
          for (int i = 0; i < nq; ++i) {
            if (P.x3d) {
              tma_load_3d(sX + q_stage[i] * xst, &P.tmX, &tail->full[q_stage[i]], 0, q_tt[i] * NN, q_k[i]);
            } else {
              for (int j = 0; j < q_nk[i]; ++j)
                tma_load_2d(sX + q_stage[i] * xst + j * xbytes, &P.tmX, &tail->full[q_stage[i]],
                            (q_k[i] + j) * kTileK, q_tt[i] * NN);
            }
          }
          nq = 0;
          ready = true;
          return true;
        };
        for (int t = w.grp; ok && t < w.tiles; t += w.ngrp) {
          const int r = t / P.tok_tiles;
          const int tt = t - r * P.tok_tiles;
          for (int kt = w.k_lo; kt < w.k_hi; kt += KPS, ++it) {
            const int nk = min(KPS, w.k_hi - kt);
            const int stage = it % S;
            const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
            // a slot still holding an earlier phase's stage frees without the grid counter; once
            // the ring holds only this phase's stages (nq == S) the counter is waited on (below)
            if (!wait_or_abort(&tail->empty[stage], ph ^ 1u, timeout_ns, tail, err)) {
              ok = false;
              break;
            }
            if (kt == w.k_lo && t == w.grp) trace_mark(A, 2 + 3 * p);
            trace_iter(A, 2, it - S);
            trace_iter(A, 0, it);
            // a 3D activation box always moves KPS k-tiles (zero-filled past the tensor)
            mbar_arrive_expect_tx(&tail->full[stage], nk * kStageW + (P.x3d ? KPS : nk) * xbytes);
            // pre-tiled weights: blocks (r, kt..kt+nk-1) are one contiguous stretch of nk x 16 KB
            // stored as the swizzled shared-memory image, so one plain bulk copy loads the stage
            if (P.w_rowmajor) {
              for (int j = 0; j < nk; ++j)
                tma_load_2d_hint(sW + stage * wst + j * kStageW, &P.tmW, &tail->full[stage],
                                 (kt + j) * kTileK, r * kTileRows, pol);
            } else {
              bulk_load_hint(sW + stage * wst,
                             static_cast<const uint8_t*>(P.W) + (static_cast<size_t>(r) * P.KT + kt) * kStageW,
                             static_cast<uint32_t>(nk * kStageW), &tail->full[stage], pol);
            }
            n_issued = it + 1;
            if (A.pf_stages > 0 && it >= S) pf_step(true);
            if (ready) {
              if (P.x3d) {
                tma_load_3d(sX + stage * xst, &P.tmX, &tail->full[stage], 0, tt * NN, kt);
              } else {
                for (int j = 0; j < nk; ++j)
                  tma_load_2d(sX + stage * xst + j * xbytes, &P.tmX, &tail->full[stage],
                              (kt + j) * kTileK, tt * NN);
              }
            } else {
              q_stage[nq] = stage;
              q_k[nq] = kt;
              q_tt[nq] = tt;
              q_nk[nq] = nk;
              if (++nq == S) {
                const bool last_k = kt + nk >= w.k_hi;
                if (!become_ready(last_k ? t + w.ngrp : t, last_k ? w.k_lo : kt + nk)) {
                  ok = false;
                  break;
                }
              }
            }
          }
        }
        if (ok && !ready && !become_ready(w.tiles, 0)) ok = false;
      }
      if (ok && A.next_valid && static_cast<int>(blockIdx.x) < A.next_grid) {
        // warm L2 (and address translation) for this CTA index's first boxes of the next chain
        const int ncl = blockIdx.x / A.next_CS;
        const int nrank = blockIdx.x % A.next_CS;
        for (int j = 0; j < 2; ++j) {
          const WarmPhase& N = A.next[j];
          if (N.boxes <= 0) continue;
          const int grp = ncl * (A.next_CS / N.s) + nrank / N.s;
          if (grp >= N.tiles) continue;
          const int nr = grp / N.tok_tiles;
          const int lo = (nrank % N.s) * N.ks;
          const int hi = min(N.KT, min(lo + N.ks, lo + N.boxes));
          if (hi > lo)
            bulk_prefetch_l2(static_cast<const uint8_t*>(N.W) + (static_cast<size_t>(nr) * N.KT + lo) * kStageW,
                             static_cast<uint32_t>((hi - lo) * kStageW));
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA can exit
        const int first = n_issued - S > 0 ? n_issued - S : 0;
        for (int j = first; j < n_issued; ++j)
          mbar_wait(&tail->full[j % S], static_cast<uint32_t>(j / S) & 1u, timeout_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA issuer --
      const uint32_t idesc = idesc_bf16_f32(kTileRows, NN);
      int it = 0, i = 0;
      bool ok = true;
      for (int p = 0; ok && p < A.nph; ++p) {
        const Work w = work_of(A, p, cl, rank, C);
        for (int t = w.grp; ok && t < w.tiles; t += w.ngrp, ++i) {
          const int tb = i & 1;
          const uint32_t use = static_cast<uint32_t>(i >> 1);
          if (!wait_or_abort(&tail->tempty[tb], (use & 1u) ^ 1u, timeout_ns, tail, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + tb * buf_cols;
          for (int kt = w.k_lo; kt < w.k_hi; kt += KPS, ++it) {
            const int nk = min(KPS, w.k_hi - kt);
            const int stage = it % S;
            const uint32_t ph = static_cast<uint32_t>(it / S) & 1u;
            if (!wait_or_abort(&tail->full[stage], ph, timeout_ns, tail, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            trace_iter(A, 1, it);
            for (int j = 0; j < nk; ++j) {
              // B reads NT token rows from an xr-row block: rows past xr are padding columns of
              // the tile (stale shared memory, never used by the epilogue)
              const uint64_t da = sdesc_k_sw128(smem_u32(sW + stage * wst + j * kStageW));
              const uint64_t db = sdesc_k_sw128(smem_u32(sX + stage * xst + j * xbytes));
#pragma unroll
              for (int kk = 0; kk < kTileK / 16; ++kk)
                tc_mma_f16(d, da + 2 * kk, db + 2 * kk, idesc, (kt > w.k_lo || j > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(&tail->empty[stage]);
          }
          if (!ok) break;
          tc_commit(&tail->tfull[tb]);
          trace_mark(A, 14);
        }
      }
    }
    __syncwarp();
    // every epilogue read of tensor memory is done once the epilogue warps reach barrier 2
    named_bar_sync(2, 32 + kEpiThreads);
    tc_fence_after();
    tmem_dealloc(tmem, A.tmem_cols);
  } else {
    // -------------------------------------------------------------------- epilogue --
    pdl_wait();
    const int et = threadIdx.x - 64;
    const int ew = warp & 3;              // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;     // which of the quarter's two warps: chunk parity
    const int row_in_tile = ew * 32 + lane;
    float* red_f = tail->red_f[half];
    int* red_i = tail->red_i[half];
    const int hbar = 3 + half;            // named barrier of this half's 4 warps
    int i = 0;    // tiles of this CTA so far (TMEM buffer parity)
    int ru = 0;   // split tiles in which this CTA owned chunks (rfull phases)
    bool ok = true;
    for (int p = 0; ok && p < A.nph; ++p) {
      const PhaseArgs& P = A.ph[p];
      const EpiArgs& e = P.e;
      const Work w = work_of(A, p, cl, rank, C);
      const bool need_norm = (e.kind != EPI_RESID);
      if (p > 0) {
        // inputs of this epilogue (residual, RMS statistics) come from phase p-1; one thread
        // polls the counter (acquire), the barrier orders the others' reads after it
        if (et == 0 && !wait_counter(A.bar + (p - 1), G, timeout_ns)) {
          tail->epi_abort = 1;
          set_err(err, NLD_DEVERR_TIMEOUT);
        }
        named_bar_sync(1, kEpiThreads);
        if (tail->epi_abort) break;
      }
      if (et == 0) trace_mark(A, 3 + 3 * p);
      const int g0 = (rank / w.s) * w.s;   // first cluster rank of this rank's group
      int kp = 0;                          // split tiles of this phase so far (same in the group)
      for (int t = w.grp; t < w.tiles; t += w.ngrp, ++i) {
        const int r = t / P.tok_tiles;
        const int tt = t - r * P.tok_tiles;
        const int tok0 = tt * NT;
        const int nvalid = min(NT, e.M - tok0);
        const int nchunks = (nvalid + 15) >> 4;
        const int tb = i & 1;
        const uint32_t use = static_cast<uint32_t>(i >> 1);
        named_bar_sync(1, kEpiThreads);
        compute_tile_meta(e, tok0, NT, need_norm, s_inv, s_pos, s_pg, s_rpos, et, kEpiThreads);
        // Split tile: the group's s ranks each hold a partial sum of the whole tile.  Rank g
        // owns chunks [g*per, (g+1)*per): every rank sends its partial of those chunks to g with
        // st.async (one-way, counted by g's rfull transaction count) and g sums the s partials
        // in rank order from its own shared memory.  Prepared while the tile's MMAs run: the
        // chunk's global operands, and the other owners' readiness for this tile.
        const int per = (nchunks + w.s - 1) / w.s;
        const int c_lo = w.grank * per, c_hi = min(nchunks, c_lo + per);
        const int n_own = max(0, c_hi - c_lo);
        // the half whose chunk parity matches reduces an owned chunk (per <= 2): the thread that
        // loads that chunk's accumulator in step 2 is the one that sums it in step 4
        const int cm = ((c_lo & 1) == half) ? c_lo : c_lo + 1;
        EpiPre pre;
        if (w.s > 1) {
          named_bar_sync(1, kEpiThreads);   // the tile's positions (QKV) are in shared memory
          if (cm < c_hi) epi_preload(e, r, row_in_tile, tok0 + cm * 16, s_rpos, cm * 16, pre);
          // every other owner of this tile has reduced the group's previous split tile of this
          // phase (earlier phases: the grid-wide phase counter), so its slots are free
          if (et < w.s && et != w.grank && et * per < nchunks) {
            const uint32_t a = dsmem_addr(smem_u32(&tail->done[p]), static_cast<uint32_t>(g0 + et));
            const uint64_t t0 = globaltimer_ns();
            while (static_cast<int>(ld_dsmem_u32_relaxed(a)) < kp) {
              if (globaltimer_ns() - t0 > timeout_ns) {
                tail->epi_abort = 1;
                set_err(err, NLD_DEVERR_TIMEOUT);
                break;
              }
            }
          }
        }
        // (epi_wait's barrier also publishes a timed-out readiness wait above)
        if (!epi_wait(&tail->tfull[tb], use & 1u, false, timeout_ns, tail, err)) { ok = false; break; }
        tc_fence_after();
        if (et == 0) trace_iter(A, 3, 8 * i);
        const uint32_t tbase = tmem + (static_cast<uint32_t>(ew * 32) << 16) + tb * buf_cols;
        if (w.s == 1) {
          for (int c = half; c < nchunks; c += 2) {
            EpiPre pre;
            epi_preload(e, r, row_in_tile, tok0 + c * 16, s_rpos, c * 16, pre);
            float v[16];
            tmem_ld_chunk(tbase, c, A.hilo, v);
            epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + c * 16, s_inv, s_pos, s_pg,
                         c * 16, v, pre, red_f, red_i, hbar);
          }
          tc_fence_before();
          mbar_arrive(&tail->tempty[tb]);
        } else {
          // 2. partial -> owners; the own chunk's partial stays in registers (v_own)
          float v_own[16];
          for (int c = half; c < nchunks; c += 2) {
            float v[16];
            tmem_ld_chunk(tbase, c, A.hilo, v);
            const int o = c / per;
            if (o == w.grank) {
#pragma unroll
              for (int j = 0; j < 16; ++j) v_own[j] = v[j];
            } else {
              const int qs = (w.grank < o) ? w.grank : w.grank - 1;   // this rank among o's senders
              const uint32_t peer = static_cast<uint32_t>(g0 + o);
              const uint32_t base = dsmem_addr(smem_u32(slots), peer) +
                                    static_cast<uint32_t>((qs * per + (c - o * per)) * kSlotFloats * 4);
              const uint32_t bar = dsmem_addr(smem_u32(&tail->rfull), peer);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                st_async_f4(base + slot_off(row_in_tile, q),
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]), bar);
            }
          }
          tc_fence_before();
          mbar_arrive(&tail->tempty[tb]);
          if (et == 0) trace_iter(A, 3, 8 * i + 1);
          // 3. the other ranks' partials of this CTA's chunks have landed
          if (n_own > 0) {
            const uint32_t rp = static_cast<uint32_t>(ru++);
            if (!epi_wait(&tail->rfull, rp & 1u, true, timeout_ns, tail, err)) { ok = false; break; }
            // arm the next owned split tile now: its senders first wait for done[] below
            if (et == 0) {
              const uint32_t nb = next_owned_bytes(A, p, t, cl, rank, C);
              if (nb) mbar_arrive_expect_tx(&tail->rfull, nb);
            }
          } else {
            named_bar_sync(1, kEpiThreads);
          }
          if (et == 0) trace_iter(A, 3, 8 * i + 2);
          // 4. reduce this thread's chunk in rank order (its own partial at its rank's place)
          if (cm < c_hi) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(slots) +
                                 static_cast<size_t>(cm - c_lo) * kSlotFloats * 4;
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            for (int q = 0; q < w.s; ++q) {
              if (q == w.grank) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] += v_own[j];
                continue;
              }
              const int qs = (q < w.grank) ? q : q - 1;
              const uint8_t* pq = src + static_cast<size_t>(qs * per) * kSlotFloats * 4;
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const float4 a4 = *reinterpret_cast<const float4*>(pq + slot_off(row_in_tile, k4));
                v[4 * k4] += a4.x;
                v[4 * k4 + 1] += a4.y;
                v[4 * k4 + 2] += a4.z;
                v[4 * k4 + 3] += a4.w;
              }
            }
            if (et == 0) trace_iter(A, 3, 8 * i + 5);
            // slot (cm - c_lo) (the first sender's partial of this half's chunk) is read only by
            // this half: once all four of its warps have summed, it is the chunk's transpose buffer
            named_bar_sync(hbar, 128);
            epi_chunk<T>(e, r, row_in_tile, lane, ew, tok0 + cm * 16, s_inv, s_pos, s_pg,
                         cm * 16, v, pre, red_f, red_i, hbar,
                         slots + static_cast<size_t>(cm - c_lo) * kSlotFloats);
            if (et == 0) trace_iter(A, 3, 8 * i + 6);
          }
          // 5. this CTA's slots are free again (relaxed: the loaded values were consumed)
          named_bar_sync(1, kEpiThreads);
          ++kp;
          if (et == 0) {
            trace_iter(A, 3, 8 * i + 3);
            st_shared_u32_relaxed_cluster(&tail->done[p], static_cast<uint32_t>(kp));
          }
        }
        if (et == 0) trace_iter(A, 3, 8 * i + 4);
      }
      if (!ok) break;
      if (et == 0) trace_mark(A, 4 + 3 * p);
      if (p + 1 < A.nph) {
        // this CTA's outputs of phase p are written: after the barrier one thread publishes
        // them (its gpu-scope fence covers the stores the barrier ordered before it) and arrives
        named_bar_sync(1, kEpiThreads);
        if (et == 0 && !(A.dbg_skip_arrive && blockIdx.x == 0 && p == 0)) {
          __threadfence();
          fence_proxy_async_global();
          red_add_release_gpu(A.bar + p, 1u);
        }
      }
    }
    tc_fence_before();
    named_bar_sync(2, 32 + kEpiThreads);
  }
  // peers may still write into this CTA's slot area or arrive on its barriers
  if (CS > 1) cluster_sync();
  __syncthreads();
  if (A.nph > 1 && threadIdx.x == 0) {
    // every thread of this CTA is past its last wait on the phase counters; the last CTA to
    // get here zeroes them (and the exit counter) for the next launch that uses them
    __threadfence();
    const unsigned old = atomicAdd(A.bar + (kMaxPhases - 1), 1u);
    if (old == G - 1) {
      for (int p = 0; p < kMaxPhases; ++p) atomicExch(A.bar + p, 0u);
      __threadfence();
    }
  }
  if (threadIdx.x == 0) trace_mark(A, 15);
}

// Dynamic shared memory of a chain launch: the ring, then the split-K slots, the tail and the
// per-column tile data.  The MMA reads NN = MMA N activation rows from each xr-row box, so the
// last box of the ring is read (nn - xr) * 128 bytes past its end: that much must still lie in
// the allocation (the bytes after the ring are read as padding columns the epilogue ignores).
size_t gemm_chain_smem_bytes(int NT, int nn, int xr, int kps, int stages, int CS, int slots) {
  const size_t stg = (CS > 1) ? static_cast<size_t>(slots) * kSlotFloats * sizeof(float) : 0;
  const size_t after = stg + sizeof(GemmTail) + static_cast<size_t>(NT) * 16;
  const size_t overread = static_cast<size_t>(nn > xr ? nn - xr : 0) * 128;
  return static_cast<size_t>(stages) * kps * (kStageW + xr * 128) + (after > overread ? after : overread);
}
int gemm_chain_max_stages() { return kMaxStages; }

cudaError_t gemm_tc_init_attributes() {
  int dev = 0, optin = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, gemm_chain_kernel<__nv_bfloat16>)) != cudaSuccess) return e;
  return cudaFuncSetAttribute(gemm_chain_kernel<__nv_bfloat16>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - static_cast<int>(fa.sharedSizeBytes));
}

// Clusters of `split` CTAs (one CTA per SM at `smem` bytes) that can be resident at once.
int gemm_tc_max_clusters(int split, size_t smem, int sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(split * (sms / split));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_chain_kernel<__nv_bfloat16>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return sms / split;
  }
  return n > 0 ? std::min(n, sms / split) : sms / split;
}

cudaError_t launch_gemm_chain(cudaStream_t st, const ChainArgs& A, int grid, uint64_t timeout_ns,
                              bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = gemm_chain_smem_bytes(A.NT, A.NT << A.hilo, A.xr, A.kps, A.stages, A.CS, A.slots);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = A.CS;
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
  return cudaLaunchKernelEx(&cfg, gemm_chain_kernel<__nv_bfloat16>, A, timeout_ns);
}

}  // namespace nld
