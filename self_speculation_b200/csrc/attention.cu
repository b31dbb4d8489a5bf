// Block-causal GQA attention over the paged KV cache.
//
// Mask (ranhao.site notes section 3.2, r9-hu digest "Method"): the m rows of a forward sit at
// positions len..len+m-1 and are cut into blocks of `block_size` starting at len; a row sees
// every cached key and every key of its own and earlier blocks: key j is visible to row p
// iff j <= len + min(floor(p/bs)*bs + bs, m) - 1.  block_size 1 is strictly causal (verify,
// AR, prefill, KV fill); block_size m is one bidirectional block (draft, diffusion).  Two
// extensions: the first causal_rows rows of every sequence are strictly causal and the blocks
// start after them (the fused diffusion fill), and a per-sequence flag (causal_seq) makes all
// rows of that sequence causal (per-sequence diffusion, where a sequence fills while the others
// denoise).  The mask is computed from these indices and never stored.
//
// Tensor-core path (bf16, head_dim 128): one CTA per (KV split, kv head, sequence x query
// tile).  Its rows are the G = Hq/Hkv query heads of that kv head times up to QT positions
// (row = position*G + head), 16 rows per warp, so K and V tiles are read once for all the
// heads that share them.  K/V tiles of 64 keys (one page) are staged by TMA with 128-byte
// swizzle in a 3-deep ring; S = Q K^T and O += P V run on mma.sync m16n8k16 (bf16 in, fp32
// accumulate); the softmax is online in registers (exp2 domain) with quad shuffles.  When the
// keys are split over several CTAs (flash decoding), those CTAs form one thread-block cluster:
// each leaves its unnormalised partial (O, running max, running sum) in its shared memory, and
// after a cluster barrier every CTA merges a slice of the rows by reading all partials over
// distributed shared memory, in split order.  No global scratch, no atomics.
#include "common.cuh"

namespace nld {

namespace {

constexpr int kMaxAttStages = 3;   // K/V ring depth: 2 or 3 (AttnArgs::stages)
constexpr int kHalfTile = kPage * 64 * 2;        // 8 KB: 64 keys x 64 dims bf16
constexpr int kKVTile = 2 * kHalfTile;           // 16 KB: 64 keys x 128 dims
constexpr int kMaxAttWarps = 9;   // rows = positions x G <= 144 (the planner's query tile).  Up
                                  // to 8 warps (two per SM sub-partition) a thread gets 255
                                  // registers; the 9-warp form (a 33-position query tile of 4
                                  // heads, many sequences) gets 168

NLD_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
NLD_DEV void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// (not volatile: a pure function of its operands, so the compiler may interleave independent
// accumulators)
NLD_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
NLD_DEV uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// The bf16 pair (x0, x1) as hi and lo halves: hi = bf16(x), lo = bf16(x - hi).
NLD_DEV void pack_bf16_hilo(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __low2float(h), x1 - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}
// Byte offset of 16-byte chunk `c` (0..15) of `row` in a [rows][128 dims] bf16 tile stored as
// two TMA boxes of 64 dims with 128-byte swizzle.
NLD_DEV uint32_t kv_off(int row, int c) {
  return static_cast<uint32_t>((c >> 3) * kHalfTile + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Last key row visible to query row p (0-based in the forward): rows p < c are strictly
// causal; the blocks of bs rows start at row c (c = 0: the plain block mask).
NLD_DEV int vis_end_of(int len, int p, int bs, int m, int c) {
  if (p < c) return len + p;
  const int blk0 = c + ((p - c) / bs) * bs;
  return len + min(blk0 + bs, m) - 1;
}

// Keys visible to row p: [0, v1] and [l2, h2] (an empty second interval unless p is a
// pre-draft row of the quadratic self-speculation forward with block k = quad_k: rows 0..k are
// the causal verify rows; row k+1+a*k+j sees the cached prefix, the verify rows 0..a, i.e. keys
// up to len+a, and the k rows of its own block at slots len+k+1+a*k ..).
NLD_DEV void row_keys(int len, int p, int bs, int m, int c, int quad_k, int& v1, int& l2, int& h2) {
  if (quad_k > 0 && p > quad_k) {
    const int blk = (p - quad_k - 1) / quad_k;
    v1 = len + blk;
    l2 = len + quad_k + 1 + blk * quad_k;
    h2 = l2 + quad_k - 1;
  } else {
    v1 = vis_end_of(len, p, bs, m, c);
    l2 = 0x7fffffff;
    h2 = -1;
  }
}
NLD_DEV bool key_visible(int key, int v1, int l2, int h2) { return key <= v1 || (key >= l2 && key <= h2); }

// 16 consecutive fp32 columns of TMEM from registers (lane = thread); visible to later tcgen05
// operations after tmem_st_wait().
NLD_DEV void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
NLD_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Wait for this thread's outstanding tcgen05.ld, with r as in-out operands so that no use of
// the loaded registers is scheduled before the wait.
NLD_DEV void tmem_ld_wait_regs(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])::"memory");
}

}  // namespace

// kHiLo (the model's forwards): q arrives in fp32 and is split into bf16 hi and lo halves, the
// probabilities P likewise, and S = (Q_hi + Q_lo) K^T, O = (P_hi + P_lo) V take two MMAs each,
// so only the bf16 K/V cache rounds; the output is written as (hi, lo) bf16 row pairs, the
// operand layout of the O projection.  Otherwise (the stand-alone entry point) q and the output
// are plain bf16 and P is rounded to bf16 for its MMA.
template <bool kHiLo, int kMaxW>
__global__ void __launch_bounds__(32 * kMaxW, 1)
    attn_mma_kernel(const __grid_constant__ CUtensorMap tmKV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  const int NS = a.stages;
  uint8_t* sV = smem + NS * kKVTile;
  uint8_t* sQ = smem + 2 * NS * kKVTile;
  uint8_t* sQl = sQ + a.NW * 16 * 256;           // lo halves of Q (kHiLo)
  // ring barriers past both the ring + query tile and the split partials that overlay them
  const int ring_q = 2 * NS * kKVTile + (kHiLo ? 2 : 1) * a.NW * 16 * 256;
  const int partials = a.NW * 16 * (128 + 2) * 4;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + max(ring_q, partials));

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nthr = blockDim.x;
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z / a.q_tiles;
  const int qt = blockIdx.z - b * a.q_tiles;
  // profiling hook: slot i of this CTA's 16 timestamps (entry 0, dependency met 1, Q staged 2,
  // KV tile t done 3+t for t < 6, partials published 10, done 11)
  auto stamp = [&](int i) {
    if (a.trace && tid == 0)
      a.trace[((static_cast<size_t>(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 16 + i] =
          globaltimer_ns();
  };
  stamp(0);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmKV);
  }
  __syncwarp();

  // The sequence length, the page table and the cached KV rows below len were written by
  // earlier forwards (kernels that completed before the one this launch may overlap: that one
  // writes only rows len..len+m-1), so the first KV tiles lying wholly in the cached prefix are
  // requested before waiting for the previous kernel.
  int len = a.lens[b];
  const int p0 = qt * a.QT;
  const int np = min(a.QT, a.m - p0);
  if (len < 0 || len + a.m > a.pps * kPage) {   // keys must stay inside the page table row
    if (tid == 0) set_err(a.err, NLD_DEVERR_KV_OVERFLOW);
    len = max(0, min(len, a.pps * kPage - a.m));
  }
  const int crow = (a.causal_seq && a.causal_seq[b]) ? a.m : a.causal_rows;
  int kv_end;
  {
    // the CTA's last row sees the furthest key (both intervals grow with the row)
    int v1, l2, h2;
    row_keys(len, p0 + np - 1, a.block_size, a.m, crow, a.quad_k, v1, l2, h2);
    kv_end = max(v1, h2) + 1;
  }
  const int n_tiles = (kv_end + kPage - 1) / kPage;
  // at least min_tiles KV tiles per split: fewer, fuller splits keep the merge short
  const int per = max(a.min_tiles, (n_tiles + a.S - 1) / a.S);
  const int t_lo = split * per;
  const int ntile = max(0, min(n_tiles, t_lo + per) - t_lo);
  __syncthreads();

  auto issue_page = [&](int i, int page) {
    const int stage = i % NS;
    const int row0 = a.layer_row0 + ((page * 2) * a.Hkv + g) * kPage;
    const int row0v = row0 + a.Hkv * kPage;
    mbar_arrive_expect_tx(&full[stage], 2 * kKVTile);
    tma_load_2d(sK + stage * kKVTile, &tmKV, &full[stage], 0, row0);
    tma_load_2d(sK + stage * kKVTile + kHalfTile, &tmKV, &full[stage], 64, row0);
    tma_load_2d(sV + stage * kKVTile, &tmKV, &full[stage], 0, row0v);
    tma_load_2d(sV + stage * kKVTile + kHalfTile, &tmKV, &full[stage], 64, row0v);
  };
  auto issue = [&](int i) { issue_page(i, a.page_table[b * a.pps + t_lo + i]); };
  // the first tiles: page ids all requested at once, before the dependency wait (the page table
  // does not change within a forward), so the tiles requested after it (the block's own keys)
  // wait on no global load; the tiles wholly in the cached prefix are requested before it
  const int n0 = min(NS, ntile);
  int n_pre = 0;
  while (n_pre < n0 && (t_lo + n_pre + 1) * kPage <= len) ++n_pre;
  int pg[kMaxAttStages];
#pragma unroll
  for (int u = 0; u < kMaxAttStages; ++u) pg[u] = (tid == 0 && u < n0) ? a.page_table[b * a.pps + t_lo + u] : 0;
  if (tid == 0) {
#pragma unroll
    for (int u = 0; u < kMaxAttStages; ++u)
      if (u < n_pre) issue_page(u, pg[u]);
  }
  __syncwarp();
  pdl_wait();
  stamp(1);
  if (tid == 0) {
#pragma unroll
    for (int u = 0; u < kMaxAttStages; ++u)
      if (u >= n_pre && u < n0) issue_page(u, pg[u]);
  }
  __syncwarp();

  // Q tile -> shared memory (row = position*G + head, 16-byte chunks XOR-swizzled by row); each
  // thread issues the global loads of kQB chunks before storing any, so they are in flight together
  const int rows_pad = a.NW * 16;
  constexpr int kQB = 8;   // 8 warps x 32 threads x 8 chunks = 128 rows x 16: one round
  for (int e0 = tid; e0 < rows_pad * 16; e0 += kQB * nthr) {
    float4 x0[kQB], x1[kQB];
    uint4 xb[kQB];
    bool ok[kQB];
#pragma unroll
    for (int u = 0; u < kQB; ++u) {
      const int e = e0 + u * nthr;
      const int r = e >> 4, c = e & 15;
      const int p = r / a.G, gq = r - p * a.G;
      ok[u] = (e < rows_pad * 16) && r < a.rows && p < np;
      x0[u] = x1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      xb[u] = make_uint4(0, 0, 0, 0);
      if (ok[u]) {
        const size_t tok = static_cast<size_t>(b) * a.m + p0 + p;
        const size_t off = ((tok * a.Hq) + g * a.G + gq) * 128 + c * 8;
        if constexpr (kHiLo) {
          const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + off);
          x0[u] = src[0];
          x1[u] = src[1];
        } else {
          xb[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + off);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kQB; ++u) {
      const int e = e0 + u * nthr;
      if (e >= rows_pad * 16) break;
      const int r = e >> 4, c = e & 15;
      uint4 val = xb[u], vlo = make_uint4(0, 0, 0, 0);
      if constexpr (kHiLo) {
        const float xs[8] = {x0[u].x, x0[u].y, x0[u].z, x0[u].w, x1[u].x, x1[u].y, x1[u].z, x1[u].w};
        split8(xs, val, vlo);
      }
      *reinterpret_cast<uint4*>(sQ + r * 256 + ((c ^ (r & 7)) << 4)) = val;
      if constexpr (kHiLo) *reinterpret_cast<uint4*>(sQl + r * 256 + ((c ^ (r & 7)) << 4)) = vlo;
    }
  }
  __syncthreads();
  stamp(2);

  // Q fragments for the warp's 16 rows, all 8 k-steps of head_dim 128 (the lo halves are
  // read from shared memory per k-step inside the tile loop)
  uint32_t qf[8][4];
  const int qr = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
  {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int c = 2 * kk + (lane >> 4);
      ldsm_x4(smem_u32(sQ + qr * 256 + ((c ^ (qr & 7)) << 4)), qf[kk][0], qf[kk][1], qf[kk][2],
              qf[kk][3]);
    }
  }
  const int ra = warp * 16 + (lane >> 2);
  const int rb = ra + 8;
  int vis_a = -1, la2 = 0x7fffffff, ha2 = -1, vis_b = -1, lb2 = 0x7fffffff, hb2 = -1;
  if (ra < a.rows && ra / a.G < np)
    row_keys(len, p0 + ra / a.G, a.block_size, a.m, crow, a.quad_k, vis_a, la2, ha2);
  if (rb < a.rows && rb / a.G < np)
    row_keys(len, p0 + rb / a.G, a.block_size, a.m, crow, a.quad_k, vis_b, lb2, hb2);

  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  bool timed_out = false;

  for (int i = 0; i < ntile; ++i) {
    const int stage = i % NS;
    if (!mbar_wait(&full[stage], static_cast<uint32_t>(i / NS) & 1u, 2000000000ull)) {
      timed_out = true;
    }
    if (__syncthreads_or(timed_out)) {
      set_err(a.err, NLD_DEVERR_TIMEOUT);
      break;
    }
    // the next kernel (a projection chain that starts by streaming weights) may launch once
    // every CTA holds its query tile and first KV tile: launched earlier, its loads queue ahead
    // of these latency-critical ones
    if (i == 0) pdl_launch_dependents();
    const int j0 = (t_lo + i) * kPage;
    const uint32_t kb = smem_u32(sK + stage * kKVTile);
    const uint32_t vb = smem_u32(sV + stage * kKVTile);

    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    // per 32 dims: the K fragments of all 8 key groups first, then the MMAs grouped so that
    // consecutive ones go to the 8 independent accumulators (each accumulator still takes its
    // terms in the order hi k-step 0, hi k-step 1, lo k-step 0, lo k-step 1)
#pragma unroll
    for (int kk2 = 0; kk2 < 4; ++kk2) {
      uint32_t kf[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int key = nt * 8 + (lane & 7);
        const int c = 4 * kk2 + (lane >> 3);
        ldsm_x4(kb + kv_off(key, c), kf[nt][0], kf[nt][1], kf[nt][2], kf[nt][3]);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(sc[nt], qf[2 * kk2], kf[nt][0], kf[nt][1]);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(sc[nt], qf[2 * kk2 + 1], kf[nt][2], kf[nt][3]);
      if constexpr (kHiLo) {
        uint32_t ql0[4], ql1[4];
        const int c0 = 4 * kk2 + (lane >> 4), c1 = c0 + 2;
        ldsm_x4(smem_u32(sQl + qr * 256 + ((c0 ^ (qr & 7)) << 4)), ql0[0], ql0[1], ql0[2], ql0[3]);
        ldsm_x4(smem_u32(sQl + qr * 256 + ((c1 ^ (qr & 7)) << 4)), ql1[0], ql1[1], ql1[2], ql1[3]);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(sc[nt], ql0, kf[nt][0], kf[nt][1]);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) mma_bf16_16816(sc[nt], ql1, kf[nt][2], kf[nt][3]);
      }
    }
    // scale, mask, online softmax (log2 domain)
    float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int key = j0 + nt * 8 + 2 * (lane & 3);
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        float s0 = sc[nt][e2] * a.scale_log2;
        float s1 = sc[nt][2 + e2] * a.scale_log2;
        if (!key_visible(key + e2, vis_a, la2, ha2)) s0 = -INFINITY;
        if (!key_visible(key + e2, vis_b, lb2, hb2)) s1 = -INFINITY;
        sc[nt][e2] = s0;
        sc[nt][2 + e2] = s1;
        mx_a = fmaxf(mx_a, s0);
        mx_b = fmaxf(mx_b, s1);
      }
    }
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
    const float base_a = (mn_a == -INFINITY) ? 0.f : mn_a;
    const float base_b = (mn_b == -INFINITY) ? 0.f : mn_b;
    const float al_a = exp2f(m_a - base_a), al_b = exp2f(m_b - base_b);
    m_a = mn_a;
    m_b = mn_b;
    float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      sc[nt][0] = exp2f(sc[nt][0] - base_a);
      sc[nt][1] = exp2f(sc[nt][1] - base_a);
      sc[nt][2] = exp2f(sc[nt][2] - base_b);
      sc[nt][3] = exp2f(sc[nt][3] - base_b);
      ps_a += sc[nt][0] + sc[nt][1];
      ps_b += sc[nt][2] + sc[nt][3];
    }
    l_a = l_a * al_a + ps_a;
    l_b = l_b * al_b + ps_b;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= al_a;
      o[n][1] *= al_a;
      o[n][2] *= al_b;
      o[n][3] *= al_b;
    }
    // O += P V
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t pa[4], pl[4];
      if constexpr (kHiLo) {
        pack_bf16_hilo(sc[2 * j][0], sc[2 * j][1], pa[0], pl[0]);
        pack_bf16_hilo(sc[2 * j][2], sc[2 * j][3], pa[1], pl[1]);
        pack_bf16_hilo(sc[2 * j + 1][0], sc[2 * j + 1][1], pa[2], pl[2]);
        pack_bf16_hilo(sc[2 * j + 1][2], sc[2 * j + 1][3], pa[3], pl[3]);
      } else {
        pa[0] = pack_bf16(sc[2 * j][0], sc[2 * j][1]);
        pa[1] = pack_bf16(sc[2 * j][2], sc[2 * j][3]);
        pa[2] = pack_bf16(sc[2 * j + 1][0], sc[2 * j + 1][1]);
        pa[3] = pack_bf16(sc[2 * j + 1][2], sc[2 * j + 1][3]);
      }
      const int key = 16 * j + (lane & 7) + ((lane >> 3) & 1) * 8;
      // the V fragments of all 128 dims first, then 16 independent accumulators per pass (each
      // takes P_hi then P_lo)
      uint32_t vf[8][4];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const int c = 2 * p + (lane >> 4);
        ldsm_x4_t(vb + kv_off(key, c), vf[p][0], vf[p][1], vf[p][2], vf[p][3]);
      }
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        mma_bf16_16816(o[2 * p], pa, vf[p][0], vf[p][1]);
        mma_bf16_16816(o[2 * p + 1], pa, vf[p][2], vf[p][3]);
      }
      if constexpr (kHiLo) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          mma_bf16_16816(o[2 * p], pl, vf[p][0], vf[p][1]);
          mma_bf16_16816(o[2 * p + 1], pl, vf[p][2], vf[p][3]);
        }
      }
    }
    __syncthreads();
    if (i < 6) stamp(3 + i);
    if (tid == 0 && i + NS < ntile) issue(i + NS);
    __syncwarp();
  }

  if (ntile == 0 || timed_out) pdl_launch_dependents();
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);

  // output row r of this CTA (part 1: the lo row of a (hi, lo) pair)
  auto out_ptr = [&](int r, int part) -> __nv_bfloat16* {
    const int p = r / a.G, gq = r - p * a.G;
    const size_t tok = static_cast<size_t>(b) * a.m + p0 + p;
    const size_t orow = kHiLo ? 2 * tok + part : tok;
    return static_cast<__nv_bfloat16*>(a.out) + orow * a.out_ld + static_cast<size_t>(g * a.G + gq) * 128;
  };
  // store the pair (x0, x1) at column d of output row r
  auto store2 = [&](int r, int d, float x0, float x1) {
    if constexpr (kHiLo) {
      uint32_t hi, lo;
      pack_bf16_hilo(x0, x1, hi, lo);
      *reinterpret_cast<uint32_t*>(out_ptr(r, 0) + d) = hi;
      *reinterpret_cast<uint32_t*>(out_ptr(r, 1) + d) = lo;
    } else {
      *reinterpret_cast<uint32_t*>(out_ptr(r, 0) + d) = pack_bf16(x0, x1);
    }
  };

  if (a.S == 1) {
    const float ia = (l_a > 0.f) ? 1.f / l_a : 0.f, ib = (l_b > 0.f) ? 1.f / l_b : 0.f;
    if (vis_a >= 0) {
#pragma unroll
      for (int n = 0; n < 16; ++n) store2(ra, n * 8 + 2 * (lane & 3), o[n][0] * ia, o[n][1] * ia);
    }
    if (vis_b >= 0) {
#pragma unroll
      for (int n = 0; n < 16; ++n) store2(rb, n * 8 + 2 * (lane & 3), o[n][2] * ib, o[n][3] * ib);
    }
    stamp(11);
    return;
  }

  // split keys: partials stay in shared memory (the K/V ring is free now), the cluster merges
  __syncthreads();
  float* sO = reinterpret_cast<float*>(sK);                  // [rows_pad][128]
  float* sML = sO + static_cast<size_t>(rows_pad) * 128;     // [rows_pad][2]
  {
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      *reinterpret_cast<float2*>(sO + ra * 128 + n * 8 + 2 * (lane & 3)) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(sO + rb * 128 + n * 8 + 2 * (lane & 3)) = make_float2(o[n][2], o[n][3]);
    }
    if ((lane & 3) == 0) {
      *reinterpret_cast<float2*>(sML + ra * 2) = make_float2(m_a, l_a);
      *reinterpret_cast<float2*>(sML + rb * 2) = make_float2(m_b, l_b);
    }
  }
  cluster_sync();
  stamp(10);
  const int S = a.S;
  const int rank = static_cast<int>(cluster_ctarank());
  const int per_rank = (a.rows + S - 1) / S;
  const int r0 = rank * per_rank, r1 = min(a.rows, r0 + per_rank);
  const uint32_t o_base = smem_u32(sO), ml_base = smem_u32(sML);
  uint32_t o_peer[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) o_peer[q] = (q < S) ? dsmem_addr(o_base, q) : 0u;
  // a warp merges one row: lane q < S reads split q's (m, l) of it and the warp shares them (the
  // cluster's shared-memory reads, which bound the merge, drop by a third)
  const uint32_t ml_lane = ((tid & 31) < S) ? dsmem_addr(ml_base, tid & 31) : 0u;
  for (int e = tid; e < (r1 - r0) * 32; e += nthr) {   // warp-uniform: nthr is whole warps
    const int r = r0 + (e >> 5), d4 = e & 31;
    const int p = r / a.G;
    if (p >= np) continue;
    // every split published (m, l) and O for every row (zeros and -inf where it saw no key),
    // so all loads are issued before any is used
    const float2 mine = (d4 < S) ? ld_dsmem_f2(ml_lane + r * 8) : make_float2(-INFINITY, 0.f);
    float2 ml[8];
    float4 ov[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      ov[q] = (q < S) ? ld_dsmem_f4(o_peer[q] + (r * 128 + d4 * 4) * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      ml[q] = make_float2(__shfl_sync(0xffffffffu, mine.x, q), __shfl_sync(0xffffffffu, mine.y, q));
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q) M = fmaxf(M, ml[q].x);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < S && ml[q].x != -INFINITY) {
        const float w = exp2f(ml[q].x - M);
        L += w * ml[q].y;
        acc.x += w * ov[q].x;
        acc.y += w * ov[q].y;
        acc.z += w * ov[q].z;
        acc.w += w * ov[q].w;
      }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    store2(r, d4 * 4, acc.x * inv, acc.y * inv);
    store2(r, d4 * 4 + 2, acc.z * inv, acc.w * inv);
  }
  stamp(11);
  cluster_sync();   // peers may still be reading this CTA's shared memory
}

// ------------------------------------------------------------------ tcgen05 attention --
// The same attention on the 5th-generation tensor cores, for query tiles of <= 128 rows: one
// CTA per (KV split, kv head, sequence x query tile), TMEM lane r = query row r.  The query tile
// sits in TMEM (packed bf16 pairs, with hi/lo both halves) as the A operand of S = Q K^T (M 128,
// N = kTile, K 128), which goes per KV tile of kTile = 64 or 128 keys (one or two pages) to one
// of two TMEM S buffers, issued up to two tiles ahead of the softmax.  kRT softmax threads per
// row (2: 8 warps, 4: 16 warps; warps w, w+4, ... share TMEM lane quarter w % 4 and an SM
// sub-partition), one per kTile/kRT-key part of each tile: a thread reads its scores, the
// threads of a row exchange their maxima through shared memory (an mbarrier per lane quarter
// and tile parity), and each writes P as packed bf16 pairs (with hi/lo: its lo half too) into
// TMEM.  O += P V (M 128, N 128, K kTile) takes P from TMEM as the A operand and V straight from
// the TMA tile as an MN-major operand.  A row's reference max moves only when a tile's max
// exceeds it by more than 2^8 (so P <= 256), which rescales its O row in TMEM (each thread
// 128/kRT columns).  Splits merge over the cluster as in attn_mma_kernel.  One thread issues
// the S MMAs; another, in another warp, loads K/V by TMA into a 192 KB ring (shared memory holds
// only the ring) and issues the P V MMAs.  TMEM columns: S buffers [0, 2 kTile), O, Q (hi pairs,
// then lo pairs); with 64-key tiles two P buffers of their own after Q, with 128-key tiles P
// over S in its buffer.
// kRT softmax threads per row (2 or 4): 128 kRT softmax threads, + the MMA warp + the TMA warp
__host__ __device__ constexpr int tc_threads(int rt) { return 128 * rt + 64; }
// KV tiles of kTile = 64 keys (one page) or 128 (two pages: S with N = 128, half the S MMAs
// per key); a ring stage holds K (and one V) of a tile, [2 dim boxes][kTile keys][128 B]; the
// ring takes 192 KB either way
constexpr int kTcMaxStages = 6;
__host__ __device__ constexpr int tc_stage_bytes(int tile) { return tile * 256; }
__host__ __device__ constexpr int tc_stages(int tile) { return tile == 64 ? 6 : 3; }
// S of tile j + 2 may be issued while tile j's stage is held: three stages at least
static_assert(tc_stages(64) >= 3 && tc_stages(128) >= 3 && tc_stages(64) <= kTcMaxStages, "ring depth");
constexpr float kTcRescale = 8.f;               // log2 units
constexpr int kTcBarBytes = 320;
// row-max exchange: [tile parity][key part][row] floats
__host__ __device__ constexpr int tc_xchg_bytes(int rt) { return 2 * rt * 128 * 4; }

// 2^x by the hardware approximation (relative error about 2^-22; 2^-inf = 0).
NLD_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 consecutive 32-bit TMEM columns from registers (lane = thread); visible to later tcgen05
// operations after tmem_st_wait().
NLD_DEV void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, bf16 inputs, fp32 accumulate; A's row i is TMEM lane i,
// two bf16 of K per 32-bit column.
NLD_DEV void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of an MN-major operand in 128-byte-swizzled atoms (64 elements of
// MN x 8 of K, 1024 bytes): `lbo` = bytes from one 64-element MN block to the next, `sbo` =
// bytes from one group of 8 K rows to the next.
NLD_DEV uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

template <bool kHiLo, int kRT, int kTile>
__global__ void __launch_bounds__(tc_threads(kRT), 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmKV, const AttnArgs a) {
  static_assert(kRT == 2 || kRT == 4, "2 or 4 softmax threads per row");
  static_assert(kTile == 64 || kTile == 128, "KV tiles of one or two pages");
  constexpr int kPg = kTile / kPage;              // pages per tile
  constexpr int kStage = tc_stage_bytes(kTile);   // K (or V) of one tile
  constexpr int kBox = kStage / 2;                // one 64-dim box of a tile: kTile rows x 128 B
  // TMEM columns: S buffers [0, 2 kTile) (P over S), O [2 kTile, 2 kTile + 128), Q after O
  constexpr uint32_t kOCol = 2 * kTile, kQCol = 2 * kTile + 128;
  // 128-key tiles write P over S (TMEM is full); 64-key tiles keep two P buffers of their own
  // after Q (columns 384..511: per buffer 32 columns of hi pairs, then 32 of lo pairs), so S of
  // tile j + 2 only waits for the softmax to have read S of tile j
  constexpr bool kAlias = kTile == 128;
  constexpr uint32_t kPCol = 2 * kTile + 256;
  constexpr int kTcSoftmax = 128 * kRT;
  constexpr int kTcThreads = tc_threads(kRT);
  constexpr int kKT = kTile / kRT;   // keys of a tile per softmax thread
  constexpr int kOC = 128 / kRT;   // O columns per softmax thread in the rescale and the combine
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int kQ = kHiLo ? 2 : 1;                // operand halves (hi, lo)
  constexpr int NS = tc_stages(kTile);
  // a stage per tile: [2 dim boxes][128 keys (page 0 rows, then page 1 rows)][128 B]
  uint8_t* sK = smem;                              // [NS] stages
  uint8_t* sV = sK + NS * kStage;                  // same
  float* xmax = reinterpret_cast<float*>(sV + NS * kStage);   // [2][kRT][128] row maxima
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + NS * kStage + tc_xchg_bytes(kRT));
  uint64_t* full = bars;              // [NS] K/V tile landed (TMA transaction bytes)
  uint64_t* empty = bars + kTcMaxStages;   // [NS] K/V stage free (the tile's P V MMAs completed)
  uint64_t* s_full = bars + 2 * kTcMaxStages;   // [2] S buffer written (MMA commit)
  // the softmax warps arrive on their barriers once per warp (lane 0, after the warp's threads
  // synchronise): one arrival per thread would queue 512 arrivals per barrier and tile
  uint64_t* s_free = s_full + 2;      // [2] S buffer read (the softmax warps; 64-key tiles)
  uint64_t* p_full = s_full + 4;      // [2] P written (the softmax warps)
  uint64_t* pv_done = s_full + 6;     // [2] O += P V from the S buffer completed (MMA commit)
  uint64_t* fin = s_full + 8;         // every MMA of both issuing threads completed
  uint64_t* xbar = s_full + 9;        // [2][4] row maxima of a lane quarter written (kRT warps)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_full + 17);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_full + 18);
  int* s_pg = reinterpret_cast<int*>(s_full + 19);   // [NS kPg] page ids of the first NS tiles
  static_assert(NS * kPg <= kTcMaxStages, "page ids of the first tiles");
  static_assert(2 * kTcMaxStages * 8 + 19 * 8 + kTcMaxStages * 4 <= kTcBarBytes, "barrier bytes");
  constexpr uint64_t kWait = 2000000000ull;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z / a.q_tiles;
  const int qt = blockIdx.z - b * a.q_tiles;
  const bool softmax_thr = tid < kTcSoftmax;
  const bool mma_thr = tid == kTcSoftmax;
  const bool tma_thr = tid == kTcSoftmax + 32;
  auto stamp = [&](int i) {
    if (a.trace && tid == 0)
      a.trace[((static_cast<size_t>(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 16 + i] =
          globaltimer_ns();
  };
  stamp(0);
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kTcSoftmax / 32);
      mbar_init(&p_full[i], kTcSoftmax / 32);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(fin, 2);   // both issuing threads commit once
    for (int i = 0; i < 8; ++i) mbar_init(&xbar[i], kRT);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmKV);
  }
  if (warp == kTcSoftmax / 32) {
    tmem_alloc(s_tmem, 512);   // S / P, O, Q (kOCol, kQCol)
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  int len = a.lens[b];
  const int p0 = qt * a.QT;
  const int np = min(a.QT, a.m - p0);
  if (len < 0 || len + a.m > a.pps * kPage) {
    if (tid == 0) set_err(a.err, NLD_DEVERR_KV_OVERFLOW);
    len = max(0, min(len, a.pps * kPage - a.m));
  }
  const int crow = (a.causal_seq && a.causal_seq[b]) ? a.m : a.causal_rows;
  int kv_end;
  {
    int v1, l2, h2;
    row_keys(len, p0 + np - 1, a.block_size, a.m, crow, a.quad_k, v1, l2, h2);
    kv_end = max(v1, h2) + 1;
  }
  // tiles of kTile keys (pages kPg t ..); the split plan's min_tiles counts pages
  const int n_pages = (kv_end + kPage - 1) / kPage;
  const int n_tiles = (n_pages + kPg - 1) / kPg;
  const int per = max((a.min_tiles + kPg - 1) / kPg, (n_tiles + a.S - 1) / a.S);
  const int t_lo = split * per;
  const int ntile = max(0, min(n_tiles, t_lo + per) - t_lo);

  int n_issued = 0;   // K/V tiles requested (TMA thread)
  // a tile's second page past the keys reads the first page again: its keys are masked, and its
  // V rows, multiplied by P = 0, must be finite
  auto page_of = [&](int i, int h) {
    const int kt = kPg * (t_lo + i);
    return a.page_table[b * a.pps + (kt + h < n_pages ? kt + h : kt)];
  };
  // the page ids of the first NS tiles, all requested at once: the page table does not change
  // within a forward, so they are read before the dependency wait, and the tiles requested
  // after it (the block's own keys) wait on no global load
  if (tma_thr) {
    const int n0 = min(NS, ntile);
    int pg[NS * kPg];
#pragma unroll
    for (int u = 0; u < NS * kPg; ++u) pg[u] = (u / kPg < n0) ? page_of(u / kPg, u % kPg) : 0;
#pragma unroll
    for (int u = 0; u < NS * kPg; ++u) s_pg[u] = pg[u];
  }
  auto issue = [&](int i) {
    ++n_issued;
    const int stage = i % NS;
    mbar_arrive_expect_tx(&full[stage], 2 * kStage);
#pragma unroll
    for (int h = 0; h < kPg; ++h) {
      const int page = i < NS ? s_pg[i * kPg + h] : page_of(i, h);
      const int row0 = a.layer_row0 + ((page * 2) * a.Hkv + g) * kPage;
      const int row0v = row0 + a.Hkv * kPage;
#pragma unroll
      for (int box = 0; box < 2; ++box) {
        tma_load_2d(sK + stage * kStage + box * kBox + h * kHalfTile, &tmKV, &full[stage], box * 64, row0);
        tma_load_2d(sV + stage * kStage + box * kBox + h * kHalfTile, &tmKV, &full[stage], box * 64, row0v);
      }
    }
  };
  // the K/V tiles wholly in the cached prefix are requested before the dependency wait
  int n_pre = 0;
  if (tma_thr)
    for (; n_pre < min(NS, ntile) && (t_lo + n_pre + 1) * kTile <= len; ++n_pre) issue(n_pre);
  pdl_wait();
  stamp(1);
  if (tma_thr)
    for (int i = n_pre; i < min(NS, ntile); ++i) issue(i);

  const int kq = tid >> 7;            // softmax threads: key part (keys kKT kq .. of a tile)
  const int r = tid & 127;            // and query row (position r / G, head r % G)
  const int prow = r / a.G;
  const bool row_ok = softmax_thr && r < a.rows && prow < np;
  // query rows -> TMEM, the A operand of S = Q K^T: thread (kq, r) writes dims kq kOC .. of row r
  // as packed bf16 pairs at columns kQCol + d / 2 (hi) and kQCol + 64 + d / 2 (lo); padding rows
  // are zero
  if (softmax_thr) {
    const uint32_t lane_q = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int gh = r - prow * a.G;
    const size_t tok = static_cast<size_t>(b) * a.m + p0 + (row_ok ? prow : 0);
    const size_t qoff = ((tok * a.Hq) + g * a.G + gh) * 128 + kq * kOC;
#pragma unroll
    for (int cc = 0; cc < kOC / 32; ++cc) {
      uint4 hv[4], lv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        hv[u] = lv[u] = make_uint4(0, 0, 0, 0);
        if (row_ok) {
          if constexpr (kHiLo) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(a.q) + qoff + cc * 32 + u * 8);
            const float4 x0 = src[0], x1 = src[1];
            const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            split8(xs, hv[u], lv[u]);
          } else {
            hv[u] = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + qoff + cc * 32 + u * 8);
          }
        }
      }
      float hw[16], lw[16];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        hw[4 * u] = __uint_as_float(hv[u].x);
        hw[4 * u + 1] = __uint_as_float(hv[u].y);
        hw[4 * u + 2] = __uint_as_float(hv[u].z);
        hw[4 * u + 3] = __uint_as_float(hv[u].w);
        lw[4 * u] = __uint_as_float(lv[u].x);
        lw[4 * u + 1] = __uint_as_float(lv[u].y);
        lw[4 * u + 2] = __uint_as_float(lv[u].z);
        lw[4 * u + 3] = __uint_as_float(lv[u].w);
      }
      tmem_st16(tmem + lane_q + kQCol + kq * (kOC / 2) + cc * 16, hw);
      if constexpr (kHiLo) tmem_st16(tmem + lane_q + kQCol + 64 + kq * (kOC / 2) + cc * 16, lw);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  stamp(2);
  pdl_launch_dependents();

  float m_ref = -INFINITY, l_sum = 0.f;
  bool aborted = false;
  // Two issuing threads, in different warps (SM sub-partitions): the MMA thread issues S = Q K^T,
  // the TMA thread loads K/V and issues O += P V.  Their MMAs touch different TMEM (S buffers /
  // O) and each commits only its own, so they need no ordering between them; splitting the
  // issue halves the per-tile issue time of the one thread that used to issue both.
  const uint32_t idS = idesc_bf16_f32(128, kTile);
  const uint32_t idO = idesc_bf16_f32(128, 128) | (1u << 16);   // B (V) MN-major
  // O += P V of tile i (P over S in S buffer i & 1, K/V stage i % NS); the stage frees when it
  // completes.  P of key part kq (keys kKT kq ..) sits in that part's S columns: kKT / 2 columns
  // of hi pairs, then kKT / 2 of lo pairs
  auto pv_step = [&](int i) -> bool {
    const int pb = i & 1, st = i % NS;
    if (*s_abort || !mbar_wait(&p_full[pb], static_cast<uint32_t>(i >> 1) & 1u, kWait)) return false;
    tc_fence_after();
#pragma unroll
    for (int q = 0; q < kQ; ++q)
#pragma unroll
      for (int ks = 0; ks < kTile / 16; ++ks) {   // 16-key step: page ks / 4, rows 16 (ks % 4) ..
        const int part = ks / (kKT / 16), u = ks % (kKT / 16);
        tc_mma_f16_ts(tmem + kOCol,
                      kAlias ? tmem + pb * kTile + part * kKT + q * (kKT / 2) + u * 8
                             : tmem + kPCol + pb * 64 + q * 32 + ks * 8,
                      sdesc_mn_sw128(smem_u32(sV + st * kStage + (ks >> 2) * kHalfTile + (ks & 3) * 2048), kBox, 1024),
                      idO, (i > 0 || q > 0 || ks > 0) ? 1u : 0u);
      }
    tc_commit(&pv_done[pb]);
    tc_commit(&empty[st]);
    return true;
  };
  // S of tile j into S buffer j & 1, free once O += P V of tile j - 2 (P over S there) completed
  auto s_step = [&](int j) -> bool {
    const int st = j % NS, sb = j & 1;
    if (*s_abort || !mbar_wait(&full[st], static_cast<uint32_t>(j / NS) & 1u, kWait) ||
        (j >= 2 && !mbar_wait(kAlias ? &pv_done[sb] : &s_free[sb], static_cast<uint32_t>((j - 2) >> 1) & 1u, kWait)))
      return false;
    tc_fence_after();
#pragma unroll
    for (int q = 0; q < kQ; ++q)
#pragma unroll
      for (int box = 0; box < 2; ++box)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16_ts(tmem + sb * kTile, tmem + kQCol + q * 64 + (box * 4 + kk) * 8,
                        sdesc_k_sw128(smem_u32(sK + st * kStage + box * kBox)) + 2 * kk, idS,
                        (q > 0 || box > 0 || kk > 0) ? 1u : 0u);
    tc_commit(&s_full[sb]);
    return true;
  };
  if (tma_thr) {
    // --------------------------------------------------------- TMA + P V thread --
    // O += P V of tile j as soon as its P is written; then tile j + NS reuses tile j's stage
    // once those MMAs have completed
    for (int j = 0; j < ntile && !aborted; ++j) {
      if (!pv_step(j)) {
        aborted = true;
        break;
      }
      if (j + NS < ntile) {
        if (!mbar_wait(&empty[j % NS], static_cast<uint32_t>(j / NS) & 1u, kWait)) {
          aborted = true;
          break;
        }
        issue(j + NS);
      }
    }
    if (aborted) {
      *s_abort = 1;
      set_err(a.err, NLD_DEVERR_TIMEOUT);
    }
    // every MMA this thread issued has completed before the tensor memory is released
    tc_commit(fin);
    mbar_wait(fin, 0, kWait);
  } else if (mma_thr) {
    // ---------------------------------------------------------------- S thread --
    // S runs up to two tiles ahead of the softmax
    for (int j = 0; j < ntile && !aborted; ++j)
      if (!s_step(j)) aborted = true;
    if (aborted) {
      *s_abort = 1;
      set_err(a.err, NLD_DEVERR_TIMEOUT);
    }
    tc_commit(fin);
    mbar_wait(fin, 0, kWait);
  } else if (softmax_thr) {
    // ------------------------------------- softmax: row r, keys kKT kq .. kKT kq + kKT - 1 --
    int v1 = -1, l2 = 0x7fffffff, h2 = -1;
    if (row_ok) row_keys(len, p0 + prow, a.block_size, a.m, crow, a.quad_k, v1, l2, h2);
    const int lq = warp & 3;   // TMEM lane quarter
    const uint32_t lane_base = static_cast<uint32_t>(lq * 32) << 16;
    const uint32_t o_col = kOCol + kq * kOC;   // this thread's columns of O
    const float c = a.scale_log2;
    for (int j = 0; j < ntile; ++j) {
      const int sb = j & 1;
      // tcgen05.ld/st are warp-collective: every exit of this loop is taken by the whole warp
      const bool ok = !*s_abort && mbar_wait(&s_full[sb], static_cast<uint32_t>(j >> 1) & 1u, kWait);
      if (!__all_sync(0xffffffffu, ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      uint32_t raw[kKT / 16][16];
#pragma unroll
      for (int u = 0; u < kKT / 16; ++u) tmem_ld16_nowait(tmem + lane_base + sb * kTile + kq * kKT + u * 16, raw[u]);
#pragma unroll
      for (int u = 0; u < kKT / 16; ++u) tmem_ld_wait_regs(raw[u]);
      if constexpr (!kAlias) {
        tc_fence_before();
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(&s_free[sb]);
      }
      float sv[kKT];
      const int k0 = (t_lo + j) * kTile + kq * kKT;
      if (k0 + kKT - 1 <= v1) {
#pragma unroll
        for (int k = 0; k < kKT; ++k) sv[k] = __uint_as_float(raw[k >> 4][k & 15]);
      } else {
#pragma unroll
        for (int k = 0; k < kKT; ++k)
          sv[k] = key_visible(k0 + k, v1, l2, h2) ? __uint_as_float(raw[k >> 4][k & 15]) : -INFINITY;
      }
      // the row's max over the tile: a tree over this thread's scores, then the kRT parts'
      // through shared memory (scores unscaled: the scale is positive)
      float mt[kKT / 2];
#pragma unroll
      for (int k = 0; k < kKT / 2; ++k) mt[k] = fmaxf(sv[k], sv[k + kKT / 2]);
#pragma unroll
      for (int w = kKT / 4; w > 0; w >>= 1)
#pragma unroll
        for (int k = 0; k < w; ++k) mt[k] = fmaxf(mt[k], mt[k + w]);
      float* xm = xmax + sb * kRT * 128;
      xm[kq * 128 + r] = mt[0];
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&xbar[sb * 4 + lq]);
      if (!__all_sync(0xffffffffu, mbar_wait(&xbar[sb * 4 + lq], static_cast<uint32_t>(j >> 1) & 1u, kWait))) {
        aborted = true;
        break;
      }
      float mx = xm[r];
#pragma unroll
      for (int q = 1; q < kRT; ++q) mx = fmaxf(mx, xm[q * 128 + r]);
      mx *= c;
      const bool move = mx > m_ref + kTcRescale;
      const bool scale_o = move && j >= 1 && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, scale_o)) {
        // the O row holds tiles < j once O += P V of tile j - 1 has completed; the warp rescales
        // its 32 rows x kOC columns together (factor 1 for rows that keep their max)
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], static_cast<uint32_t>((j - 1) >> 1) & 1u, kWait))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const float alpha = scale_o ? exp2f(m_ref - mx) : 1.f;
#pragma unroll
        for (int cc = 0; cc < kOC / 16; ++cc) {
          float o[16];
          tmem_ld16(tmem + lane_base + o_col + cc * 16, o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] *= alpha;
          tmem_st16(tmem + lane_base + o_col + cc * 16, o);
        }
        tmem_st_wait();
        l_sum *= alpha;
      }
      if (move) m_ref = mx;
      const float nb = (m_ref == -INFINITY) ? 0.f : -m_ref;
      // P row r, this thread's keys as kKT / 2 bf16 pairs (lower key in the low half), hi then lo
      uint32_t ph[kKT / 16][8], pl[kKT / 16][8];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < kKT / 2; ++k) {
        const float q0 = ex2_approx(fmaf(sv[2 * k], c, nb)), q1 = ex2_approx(fmaf(sv[2 * k + 1], c, nb));
        ls[k & 3] += q0 + q1;
        if constexpr (kHiLo) {
          pack_bf16_hilo(q0, q1, ph[k >> 3][k & 7], pl[k >> 3][k & 7]);
        } else {
          ph[k >> 3][k & 7] = pack_bf16(q0, q1);
          pl[k >> 3][k & 7] = 0u;
        }
      }
      l_sum += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      // P: 128-key tiles over this thread's own S columns (read above), kKT / 2 columns of hi
      // pairs then lo; 64-key tiles into P buffer sb
      // 64-key tiles: P buffer sb is free once O += P V of tile j - 2 has completed
      if constexpr (!kAlias) {
        if (!__all_sync(0xffffffffu, j < 2 || mbar_wait(&pv_done[sb], static_cast<uint32_t>((j - 2) >> 1) & 1u, kWait))) {
          aborted = true;
          break;
        }
      }
      const uint32_t p_col = kAlias ? sb * kTile + kq * kKT : kPCol + sb * 64 + kq * (kKT / 2);
      const uint32_t p_lo = kAlias ? kKT / 2 : 32;   // lo pairs after the hi pairs
#pragma unroll
      for (int u = 0; u < kKT / 16; ++u) {
        tmem_st8(tmem + lane_base + p_col + u * 8, ph[u]);
        if constexpr (kHiLo) tmem_st8(tmem + lane_base + p_col + p_lo + u * 8, pl[u]);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&p_full[sb]);
      if (j < 6 && tid == 0) stamp(3 + j);
    }
    if (!aborted && ntile > 0 &&
        !__all_sync(0xffffffffu, mbar_wait(&pv_done[(ntile - 1) & 1], static_cast<uint32_t>((ntile - 1) >> 1) & 1u, kWait)))
      aborted = true;
    if (aborted) {
      *s_abort = 1;
      set_err(a.err, NLD_DEVERR_TIMEOUT);
    }
    tc_fence_after();
    stamp(12);
  }

  // output row rr of this CTA (part 1: the lo row of a (hi, lo) pair)
  auto out_ptr = [&](int rr, int part) -> __nv_bfloat16* {
    const int p = rr / a.G, gh = rr - p * a.G;
    const size_t tok = static_cast<size_t>(b) * a.m + p0 + p;
    const size_t orow = kHiLo ? 2 * tok + part : tok;
    return static_cast<__nv_bfloat16*>(a.out) + orow * a.out_ld + static_cast<size_t>(g * a.G + gh) * 128;
  };
  auto store2 = [&](int rr, int d, float x0, float x1) {
    if constexpr (kHiLo) {
      uint32_t hi, lo;
      pack_bf16_hilo(x0, x1, hi, lo);
      *reinterpret_cast<uint32_t*>(out_ptr(rr, 0) + d) = hi;
      *reinterpret_cast<uint32_t*>(out_ptr(rr, 1) + d) = lo;
    } else {
      *reinterpret_cast<uint32_t*>(out_ptr(rr, 0) + d) = pack_bf16(x0, x1);
    }
  };

  // the CTA's partial (O unnormalised, (m, L)) into shared memory: the kRT key parts' row sums
  // add up (one reference max per row), thread (q, r) moves columns kOC q .. of O; float4 slot s
  // of row r sits at slot s ^ (r % 32)
  __syncthreads();   // every MMA and every TMA load of this CTA has completed
  float* sO = reinterpret_cast<float*>(smem);            // [128][128] partials (over Q, K)
  float* sML = sO + 128 * 128;                           // [128][2]
  float* sLq = sML + 256;                                // [kRT][128] row sums per key part
  const bool have = ntile > 0 && !*s_abort;
  // after a timeout anywhere, the loads still in flight land before the ring is overlaid
  if (tma_thr && !have)
    for (int t = max(0, n_issued - NS); t < n_issued; ++t)
      mbar_wait(&full[t % NS], static_cast<uint32_t>(t / NS) & 1u, kWait);
  if (softmax_thr) sLq[kq * 128 + r] = have ? l_sum : 0.f;
  __syncthreads();
  if (softmax_thr) {
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
#pragma unroll
    for (int cc = 0; cc < kOC / 32; ++cc) {
      uint32_t o[2][16];
      if (have) {
        tmem_ld16_nowait(tmem + lane_base + kOCol + kq * kOC + cc * 32, o[0]);
        tmem_ld16_nowait(tmem + lane_base + kOCol + kq * kOC + cc * 32 + 16, o[1]);
        tmem_ld_wait_regs(o[0]);
        tmem_ld_wait_regs(o[1]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) o[0][i] = o[1][i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const int slot = ((kq * kOC + cc * 32 + i) >> 2) ^ (r & 31);
        *reinterpret_cast<float4*>(sO + r * 128 + slot * 4) =
            make_float4(__uint_as_float(o[i >> 4][i & 15]), __uint_as_float(o[i >> 4][(i & 15) + 1]),
                        __uint_as_float(o[i >> 4][(i & 15) + 2]), __uint_as_float(o[i >> 4][(i & 15) + 3]));
      }
    }
    if (kq == 0) {
      float L = 0.f;
#pragma unroll
      for (int q = 0; q < kRT; ++q) L += sLq[q * 128 + r];
      *reinterpret_cast<float2*>(sML + r * 2) = make_float2(have ? m_ref : -INFINITY, L);
    }
  }
  tc_fence_before();
  __syncthreads();
  stamp(13);
  if (warp == kTcSoftmax / 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the S splits' partials merge: rank q of the cluster writes rows [q rows/S, (q+1) rows/S),
  // one warp per row, each thread 4 dims (coalesced output)
  const int S = a.S;
  if (S > 1) cluster_sync();
  stamp(10);
  const int rank = static_cast<int>(cluster_ctarank());
  const int per_rank = (a.rows + S - 1) / S;
  const int r0 = rank * per_rank, r1 = min(a.rows, r0 + per_rank);
  const uint32_t o_base = smem_u32(sO), ml_base = smem_u32(sML);
  uint32_t o_peer[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) o_peer[q] = (q < S) ? dsmem_addr(o_base, q) : 0u;
  // a warp merges one row: lane q < S reads split q's (m, L) of it and the warp shares them (the
  // cluster's shared-memory reads, which bound the merge, drop by a third)
  const uint32_t ml_lane = ((tid & 31) < S) ? dsmem_addr(ml_base, tid & 31) : 0u;
  for (int e = tid; e < (r1 - r0) * 32; e += kTcThreads) {   // warp-uniform
    const int rr = r0 + (e >> 5), d4 = e & 31;
    if (rr / a.G >= np) continue;
    const uint32_t o_off = (rr * 128 + ((d4 ^ (rr & 31)) << 2)) * 4;
    const float2 mine = (d4 < S) ? ld_dsmem_f2(ml_lane + rr * 8) : make_float2(-INFINITY, 0.f);
    float2 ml[8];
    float4 ov[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) ov[q] = (q < S) ? ld_dsmem_f4(o_peer[q] + o_off) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      ml[q] = make_float2(__shfl_sync(0xffffffffu, mine.x, q), __shfl_sync(0xffffffffu, mine.y, q));
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q) M = fmaxf(M, ml[q].x);
    float L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < S && ml[q].x != -INFINITY) {
        const float w = exp2f(ml[q].x - M);
        L += w * ml[q].y;
        acc.x += w * ov[q].x;
        acc.y += w * ov[q].y;
        acc.z += w * ov[q].z;
        acc.w += w * ov[q].w;
      }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    if (e == tid) stamp(14);
    store2(rr, d4 * 4, acc.x * inv, acc.y * inv);
    store2(rr, d4 * 4 + 2, acc.z * inv, acc.w * inv);
  }
  stamp(11);
  if (S > 1) cluster_sync();   // peers may still be reading this CTA's shared memory
}

// Plain per-(token, head) attention for any head_dim <= 128 and either storage type; used by
// the fp32 configuration.  Scores go to shared memory (max_kv floats), two-pass softmax.
template <typename T>
__global__ void __launch_bounds__(128) attn_simt_kernel(const AttnArgs a) {
  extern __shared__ float sm[];
  float* sq = sm;             // [hd]
  float* sc = sm + 128;       // [max_kv]
  __shared__ float red[4];
  pdl_wait();
  pdl_launch_dependents();
  const int tok = blockIdx.x, head = blockIdx.y;
  const int b = tok / a.m, i = tok - b * a.m;
  const int g = head / a.G;
  int len = a.lens[b];
  if (len < 0 || len + a.m > a.pps * kPage) {
    if (threadIdx.x == 0) set_err(a.err, NLD_DEVERR_KV_OVERFLOW);
    len = max(0, min(len, a.pps * kPage - a.m));
  }
  const int crow = (a.causal_seq && a.causal_seq[b]) ? a.m : a.causal_rows;
  int v1, l2, h2;
  row_keys(len, i, a.block_size, a.m, crow, a.quad_k, v1, l2, h2);
  const int nkeys = max(v1, h2) + 1;
  const T* q = static_cast<const T*>(a.q) + (static_cast<size_t>(tok) * a.Hq + head) * a.hd;
  for (int d = threadIdx.x; d < a.hd; d += blockDim.x) sq[d] = to_f32<T>(q[d]);
  __syncthreads();
  const T* pool = static_cast<const T*>(a.pool);
  const float scale = rsqrtf(static_cast<float>(a.hd));
  for (int j = threadIdx.x; j < nkeys; j += blockDim.x) {
    const int page = a.page_table[b * a.pps + (j >> 6)];
    const T* kr = pool + ((static_cast<size_t>(page) * 2) * a.Hkv + g) * kPage * a.hd +
                  static_cast<size_t>(j & 63) * a.hd;
    float acc = 0.f;
    for (int d = 0; d < a.hd; ++d) acc += sq[d] * to_f32<T>(kr[d]);
    sc[j] = key_visible(j, v1, l2, h2) ? acc * scale : -INFINITY;
  }
  __syncthreads();
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < nkeys; j += blockDim.x) mx = fmaxf(mx, sc[j]);
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  float sum = 0.f;
  for (int j = threadIdx.x; j < nkeys; j += blockDim.x) {
    const float p = expf(sc[j] - mx);
    sc[j] = p;
    sum += p;
  }
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  sum = ((red[0] + red[1]) + red[2]) + red[3];
  const float inv = 1.f / sum;
  T* out = static_cast<T*>(a.out) + (static_cast<size_t>(tok) * a.Hq + head) * a.hd;
  for (int d = threadIdx.x; d < a.hd; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < nkeys; ++j) {
      const int page = a.page_table[b * a.pps + (j >> 6)];
      const T* vr = pool + ((static_cast<size_t>(page) * 2 + 1) * a.Hkv + g) * kPage * a.hd +
                    static_cast<size_t>(j & 63) * a.hd;
      acc += sc[j] * to_f32<T>(vr[d]);
    }
    out[d] = from_f32<T>(acc * inv);
  }
}

cudaError_t gemm_tc_init_attributes();

namespace {
using AttnKernel = void (*)(const CUtensorMap, const AttnArgs);
// The instantiation for a launch: tcgen05 or mma.sync, its operand form and (mma.sync) its
// launch bound (<= 8 or 9 warps).
AttnKernel attn_kernel_for(bool hilo, int NW, int tc, int tile) {
  if (tc && tile == 64) {
    if (tc == 2) return hilo ? attn_tc_kernel<true, 2, 64> : attn_tc_kernel<false, 2, 64>;
    return hilo ? attn_tc_kernel<true, 4, 64> : attn_tc_kernel<false, 4, 64>;
  }
  if (tc == 2) return hilo ? attn_tc_kernel<true, 2, 128> : attn_tc_kernel<false, 2, 128>;
  if (tc) return hilo ? attn_tc_kernel<true, 4, 128> : attn_tc_kernel<false, 4, 128>;
  if (NW > 8) return hilo ? attn_mma_kernel<true, 9> : attn_mma_kernel<false, 9>;
  return hilo ? attn_mma_kernel<true, 8> : attn_mma_kernel<false, 8>;
}
}  // namespace

// Shared-memory opt-ins of the large-smem kernels (host, once per process and device).
cudaError_t init_kernel_attributes() {
  cudaError_t e = gemm_tc_init_attributes();
  if (e != cudaSuccess) return e;
  int dev = 0, optin = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  // mma.sync (hilo x 8/9 warps), tcgen05 (hilo x 2/4 per row x 64/128-key tiles)
  for (int v = 0; v < 12; ++v) {
    const AttnKernel k = attn_kernel_for(v & 1, (v & 2) ? 9 : 8, v >= 4 ? 2 * ((v >> 1) & 1) + 2 : 0, v >= 8 ? 64 : 128);
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, k)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  optin - static_cast<int>(fa.sharedSizeBytes))) != cudaSuccess)
      return e;
  }
  return cudaSuccess;
}

// Dynamic shared memory of a launch: the K/V ring and the query tile (hi and lo halves with
// hilo), then the ring's barriers; the split partials (fp32 O and (m, l) per row) overlay the
// ring and the query tile once the KV loop is done.
size_t attn_mma_smem_bytes(int NW, bool hilo, int stages) {
  const size_t ring_q = 2 * static_cast<size_t>(stages) * kKVTile + static_cast<size_t>(hilo ? 2 : 1) * NW * 16 * 256;
  const size_t partials = static_cast<size_t>(NW) * 16 * (128 + 2) * sizeof(float);
  return 1024 + std::max(ring_q, partials) + kMaxAttStages * sizeof(uint64_t);
}

// Dynamic shared memory of a tcgen05 attention launch: the K and V rings (the query tile lives in
// TMEM), the row-max exchange and the barriers; the split partials overlay the rings after the
// KV loop.
size_t attn_tc_smem_bytes(bool, int rt) {
  // the same ring bytes for either tile size
  return 1024 + 2 * static_cast<size_t>(tc_stages(128)) * tc_stage_bytes(128) + tc_xchg_bytes(rt) + kTcBarBytes;
}

// Clusters of S CTAs (NW warps, the shared memory above; or the tcgen05 kernel) that can be
// resident at once.
int attn_mma_max_clusters(int S, int NW, bool hilo, int stages, int sms, int tc) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S * (sms / S));
  cfg.blockDim = dim3(tc ? tc_threads(tc) : 32 * NW);
  cfg.dynamicSmemBytes = tc ? attn_tc_smem_bytes(hilo, tc) : attn_mma_smem_bytes(NW, hilo, stages);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, attn_kernel_for(hilo, NW, tc, 128), &cfg);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return sms / S;
  }
  return n > 0 ? n : 1;
}

cudaError_t launch_attention_mma(cudaStream_t st, const CUtensorMap* tmKV, const AttnArgs& a,
                                 int batch, bool pdl) {
  const int tc = a.tc;
  if ((tc != 0 && tc != 2 && tc != 4) ||
      (tc ? (a.rows < 1 || a.rows > 128 || a.S < 1 || a.S > 8 || (a.tc_tile != 64 && a.tc_tile != 128))
          : (a.NW < 1 || a.NW > kMaxAttWarps || a.stages < 2 || a.stages > kMaxAttStages)))
    return cudaErrorInvalidValue;   // kernel form, tile rows / launch bound, ring depth
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.S, a.Hkv, batch * a.q_tiles);
  cfg.blockDim = dim3(tc ? tc_threads(tc) : 32 * a.NW);
  cfg.dynamicSmemBytes = tc ? attn_tc_smem_bytes(a.hilo != 0, tc) : attn_mma_smem_bytes(a.NW, a.hilo != 0, a.stages);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = a.S;
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) attrs[na++] = attr[0];
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_kernel_for(a.hilo != 0, a.NW, tc, a.tc_tile), *tmKV, a);
}

cudaError_t launch_attention_simt(cudaStream_t st, const AttnArgs& a, int batch, bool f32,
                                  int max_kv, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(batch * a.m, a.Hq);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = (128 + static_cast<size_t>(max_kv)) * sizeof(float);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (f32) return cudaLaunchKernelEx(&cfg, attn_simt_kernel<float>, a);
  return cudaLaunchKernelEx(&cfg, attn_simt_kernel<__nv_bfloat16>, a);
}

}  // namespace nld
