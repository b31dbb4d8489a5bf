// Fused epilogues of the projection GEMMs.  One thread owns one weight row (one output
// feature) of a 128-row tile and 16 token columns of the accumulator.  The weight rows are
// stored so that the two values an epilogue pairs sit in adjacent rows (lanes l and l^1):
//   q/k rows of a head: row 2i = feature i, row 2i+1 = feature i + hd/2 (RoPE rotate-half
//                       pairs; notes section 5 model: Llama-style RoPE);
//   gate/up tile t:     row 2i = gate feature 64t+i, row 2i+1 = up feature 64t+i (SwiGLU).
// so a single __shfl_xor(.., 1) brings the partner value.
#pragma once

#include "common.cuh"

namespace nld {

// Per-column data of a tile, computed once per tile into shared memory (see
// compute_tile_meta): s_inv = 1/rms of the token, s_pos = its KV slot (-1: no KV row: column
// past M or past the KV capacity), s_pg = the KV page holding that slot, s_rpos = its RoPE
// position (the slot itself except in the quadratic self-speculation forward).
// red_f / red_i: shared scratch of at least 4*16 + 16 entries each, private to the 4 warps (one
// per TMEM lane quarter, 128 threads) that call this together and synchronise on named
// barrier `bar_id`.
// The global operands of a 16-column chunk (epi_preload) are loaded together, ahead of the
// accumulator values where the caller can (a split tile loads them before waiting for its
// group's partials), so a chunk costs at most one memory round trip.
struct EpiPre {
  float a[16];   // EPI_RESID: residual h of the 16 tokens; EPI_QKV: RoPE cos (even feature
                 // rows) or sin (odd rows) of each token: the pair's other thread holds the other
};

NLD_DEV void qkv_row_info(const EpiArgs& e, int row, int& sec, int& head, int& lr, int& feat) {
  const int qd = e.Hq * e.hd, kvd = e.Hkv * e.hd;
  int base;
  if (row < qd) {
    sec = 0; base = 0;
  } else if (row < qd + kvd) {
    sec = 1; base = qd;
  } else {
    sec = 2; base = qd + kvd;
  }
  const int rr = row - base;
  head = rr / e.hd;
  lr = rr - head * e.hd;
  const int half = e.hd >> 1;
  feat = (sec == 2) ? lr : ((lr & 1) ? (lr >> 1) + half : (lr >> 1));
}

NLD_DEV void epi_preload(const EpiArgs& e, int row_tile, int row_in_tile, int tok0,
                         const int* s_rpos, int col0, EpiPre& p) {
  const int row = row_tile * kTileRows + row_in_tile;
  if (e.kind == EPI_RESID) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      p.a[j] = (tok0 + j < e.M) ? e.h[static_cast<size_t>(tok0 + j) * e.d + row] : 0.f;
  } else if (e.kind == EPI_QKV) {
    int sec, head, lr, feat;
    qkv_row_info(e, row, sec, head, lr, feat);
    const int half = e.hd >> 1;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int pos = s_rpos[col0 + j];
      p.a[j] = (sec < 2 && pos >= 0)
                   ? __ldg(reinterpret_cast<const float*>(&e.rope[static_cast<size_t>(pos) * half + (lr >> 1)]) +
                           (lr & 1))
                   : ((lr & 1) ? 0.f : 1.f);
    }
  }
}

// Eight fp32 values as one 16-byte piece of bf16 (round to nearest even).
NLD_DEV uint4 pack8_bf16(const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 v = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    w[q] = *reinterpret_cast<uint32_t*>(&v);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Store of one bf16 activation value: with hi/lo operands (hl) the row pair (2 tok, 2 tok + 1)
// of a [2 M, ld] buffer receives bf16(x) and bf16(x - bf16(x)); otherwise row tok of [M, ld].
template <typename T>
NLD_DEV void store_act(void* buf, bool hl, int tok, int ld, int col, float x) {
  if (hl) {
    __nv_bfloat16 hi, lo;
    split_bf16(x, hi, lo);
    __nv_bfloat16* b = static_cast<__nv_bfloat16*>(buf);
    b[static_cast<size_t>(2 * tok) * ld + col] = hi;
    b[static_cast<size_t>(2 * tok + 1) * ld + col] = lo;
  } else {
    static_cast<T*>(buf)[static_cast<size_t>(tok) * ld + col] = from_f32<T>(x);
  }
}
// Same for eight consecutive values (one 16-byte piece per stored row; bf16 storage only).
NLD_DEV void store_act8(void* buf, bool hl, int tok, int ld, int col, const float* x) {
  __nv_bfloat16* b = static_cast<__nv_bfloat16*>(buf);
  if (hl) {
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(b + static_cast<size_t>(2 * tok) * ld + col) = hi;
    *reinterpret_cast<uint4*>(b + static_cast<size_t>(2 * tok + 1) * ld + col) = lo;
  } else {
    *reinterpret_cast<uint4*>(b + static_cast<size_t>(tok) * ld + col) = pack8_bf16(x);
  }
}

// Every per-column loop below runs stage by stage over all 16 columns (all loads, then all
// multiplies, then all shuffles of one butterfly level, ...): a column-at-a-time loop is a
// chain of dependent shared-memory and shuffle latencies 16 times over (~1.3-2 us per chunk
// measured), while the stage-wise form keeps 16 independent operations in flight.
//
// Vector stores (xbuf != nullptr, bf16 storage, 128-row tiles aligned to heads): the 128
// threads first write the chunk's fp32 outputs transposed, [16 tokens][row], into xbuf (16 x
// 128 floats, private to these 4 warps), then each thread stores whole 16-byte pieces of token
// rows.  With hi/lo activations (e.hilo) the bf16 activation outputs (hb, u) are written as
// row pairs (hi, lo) and q is kept in fp32.
template <typename T>
NLD_DEV void epi_chunk(const EpiArgs& e, int row_tile, int row_in_tile, int lane, int ew,
                       int tok0, const float* s_inv, const int* s_pos, const int* s_pg, int col0,
                       float (&v)[16], const EpiPre& pre, float* red_f, int* red_i, int bar_id,
                       float* xbuf = nullptr) {
  const int row = row_tile * kTileRows + row_in_tile;
  constexpr int kXld = 128;   // floats per token row of xbuf (one split-K slot: 16 x 128 floats)
  const bool vec = (xbuf != nullptr) && sizeof(T) == 2;
  const bool hl = (sizeof(T) == 2) && e.hilo;
  switch (e.kind) {
    case EPI_QKV: {
      int sec, head, lr, feat;
      qkv_row_info(e, row, sec, head, lr, feat);
      float x[16], pt[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = s_inv[col0 + j];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] *= v[j];
#pragma unroll
      for (int j = 0; j < 16; ++j) pt[j] = __shfl_xor_sync(0xffffffffu, x[j], 1);
      if (sec < 2) {
        // rows 2i and 2i+1 (lanes l, l^1) rotate the same pair; each thread holds one of the
        // pair's (cos, sin) and takes the other from its partner
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float other = __shfl_xor_sync(0xffffffffu, pre.a[j], 1);
          const float c = (lr & 1) ? other : pre.a[j], sn = (lr & 1) ? pre.a[j] : other;
          x[j] = (lr & 1) ? (x[j] * c + pt[j] * sn) : (x[j] * c - pt[j] * sn);
        }
      }
      if (vec && e.hd == kTileRows) {
        // one tile = one head of q, k or v: the token's 128 features are one row of xbuf
#pragma unroll
        for (int j = 0; j < 16; ++j) xbuf[j * kXld + feat] = x[j];
        named_bar_sync(bar_id, 128);
        if (row_tile * kTileRows >= e.n_rows) break;
        if (sec == 0 && hl) {
          // q in fp32: 16 tokens x 32 pieces of 4 floats
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int idx = row_in_tile + 128 * q;
            const int j = idx >> 5, c4 = idx & 31;
            const int tok = tok0 + j;
            if (tok < e.M)
              *reinterpret_cast<float4*>(static_cast<float*>(e.q_out) +
                                         (static_cast<size_t>(tok) * e.Hq + head) * e.hd + c4 * 4) =
                  *reinterpret_cast<const float4*>(xbuf + j * kXld + c4 * 4);
          }
          break;
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int idx = row_in_tile + 128 * q;
          const int j = idx >> 4, c8 = idx & 15;
          const int tok = tok0 + j;
          if (tok >= e.M) continue;
          const uint4 val = pack8_bf16(xbuf + j * kXld + c8 * 8);
          if (sec == 0) {
            *reinterpret_cast<uint4*>(static_cast<T*>(e.q_out) +
                                      (static_cast<size_t>(tok) * e.Hq + head) * e.hd + c8 * 8) = val;
          } else {
            const int pos = s_pos[col0 + j];
            if (pos < 0) continue;
            const size_t off =
                ((static_cast<size_t>(s_pg[col0 + j]) * 2 + (sec - 1)) * e.Hkv + head) * kPage * e.hd +
                static_cast<size_t>(pos & (kPage - 1)) * e.hd + c8 * 8;
            *reinterpret_cast<uint4*>(static_cast<T*>(e.kv_layer) + off) = val;
          }
        }
        break;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int tok = tok0 + j;
        if (tok >= e.M || row >= e.n_rows) continue;
        if (sec == 0) {
          const size_t qi = (static_cast<size_t>(tok) * e.Hq + head) * e.hd + feat;
          if (hl)
            static_cast<float*>(e.q_out)[qi] = x[j];
          else
            static_cast<T*>(e.q_out)[qi] = from_f32<T>(x[j]);
        } else {
          const int pos = s_pos[col0 + j];
          if (pos < 0) continue;
          const size_t off =
              ((static_cast<size_t>(s_pg[col0 + j]) * 2 + (sec - 1)) * e.Hkv + head) * kPage * e.hd +
              static_cast<size_t>(pos & (kPage - 1)) * e.hd + feat;
          static_cast<T*>(e.kv_layer)[off] = from_f32<T>(x[j]);
        }
      }
    } break;

    case EPI_RESID: {
      float hn[16], sq[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) hn[j] = (tok0 + j < e.M) ? pre.a[j] + v[j] : 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (tok0 + j >= e.M) continue;
        if (vec) {
          xbuf[j * kXld + row_in_tile] = hn[j];
        } else {
          e.h[static_cast<size_t>(tok0 + j) * e.d + row] = hn[j];
          store_act<T>(e.hb, hl, tok0 + j, e.d, row, hn[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) sq[j] = hn[j] * hn[j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) sq[j] += __shfl_xor_sync(0xffffffffu, sq[j], off);
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red_f[ew * 16 + j] = sq[j];
      }
      named_bar_sync(bar_id, 128);
      if (row_in_tile < 16) {
        const int j = row_in_tile;
        const int tok = tok0 + j;
        if (tok < e.M) {
          const float s = ((red_f[j] + red_f[16 + j]) + red_f[32 + j]) + red_f[48 + j];
          e.ssq_out[static_cast<size_t>(row_tile) * e.ssq_ld + tok] = s;
        }
      }
      if (vec && row_tile * kTileRows < e.n_rows) {
        // h: 16 tokens x 128 fp32 = 512 16-byte pieces; hb: 256 pieces of 8 bf16 per stored row
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int idx = row_in_tile + 128 * q;
          const int j = idx >> 5, c4 = idx & 31;
          if (tok0 + j < e.M)
            *reinterpret_cast<float4*>(e.h + static_cast<size_t>(tok0 + j) * e.d + row_tile * kTileRows + c4 * 4) =
                *reinterpret_cast<const float4*>(xbuf + j * kXld + c4 * 4);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int idx = row_in_tile + 128 * q;
          const int j = idx >> 4, c8 = idx & 15;
          if (tok0 + j < e.M)
            store_act8(e.hb, hl, tok0 + j, e.d, row_tile * kTileRows + c8 * 8, xbuf + j * kXld + c8 * 8);
        }
      }
      named_bar_sync(bar_id, 128);
    } break;

    case EPI_SWIGLU: {
      const int f = row_tile * (kTileRows / 2) + (row_in_tile >> 1);
      float x[16], pt[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = s_inv[col0 + j];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] *= v[j];
#pragma unroll
      for (int j = 0; j < 16; ++j) pt[j] = __shfl_xor_sync(0xffffffffu, x[j], 1);
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = __fdividef(x[j], 1.0f + __expf(-x[j])) * pt[j];   // silu(g) * u
      if (vec) {
        // 16 tokens x 64 outputs: one 16-byte piece (per stored row) per thread
        if (!(lane & 1)) {
#pragma unroll
          for (int j = 0; j < 16; ++j) xbuf[j * kXld + (row_in_tile >> 1)] = x[j];
        }
        named_bar_sync(bar_id, 128);
        const int j = row_in_tile >> 3, c8 = row_in_tile & 7;
        if (tok0 + j < e.M && row_tile * kTileRows < e.n_rows)
          store_act8(e.u_out, hl, tok0 + j, e.F, row_tile * (kTileRows / 2) + c8 * 8, xbuf + j * kXld + c8 * 8);
        break;
      }
      if (!(lane & 1)) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (tok0 + j < e.M) store_act<T>(e.u_out, hl, tok0 + j, e.F, f, x[j]);
      }
    } break;

    case EPI_LOGITS: {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int tok = tok0 + j;
        if (tok < e.M && row < e.V)
          e.logits[static_cast<size_t>(tok) * e.V + row] = v[j] * s_inv[col0 + j];
      }
    } break;

    case EPI_LMHEAD: {
      // pass 1: per column max and lowest argmax over the tile's 128 rows
      float l[16], mx[16];
      int ix[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) l[j] = s_inv[col0 + j];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        l[j] = (row < e.V) ? v[j] * l[j] : -INFINITY;
        mx[j] = l[j];
        ix[j] = row;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float omx = __shfl_xor_sync(0xffffffffu, mx[j], off);
          const int oix = __shfl_xor_sync(0xffffffffu, ix[j], off);
          if (omx > mx[j] || (omx == mx[j] && oix < ix[j])) {
            mx[j] = omx;
            ix[j] = oix;
          }
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          red_f[ew * 16 + j] = mx[j];
          red_i[ew * 16 + j] = ix[j];
        }
      }
      named_bar_sync(bar_id, 128);
      if (row_in_tile < 16) {
        const int j = row_in_tile;
        float m = red_f[j];
        int x = red_i[j];
#pragma unroll
        for (int w = 1; w < 4; ++w) {
          const float o = red_f[w * 16 + j];
          if (o > m) {   // earlier warps hold lower rows: strict > keeps the lowest index
            m = o;
            x = red_i[w * 16 + j];
          }
        }
        red_f[64 + j] = m;
        red_i[64 + j] = x;
      }
      named_bar_sync(bar_id, 128);
      // pass 2: sum over the tile of exp(l - tile max)
      float sm[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sm[j] = red_f[64 + j];
#pragma unroll
      for (int j = 0; j < 16; ++j) sm[j] = (l[j] == -INFINITY) ? 0.f : expf(l[j] - sm[j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int j = 0; j < 16; ++j) sm[j] += __shfl_xor_sync(0xffffffffu, sm[j], off);
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) red_f[ew * 16 + j] = sm[j];
      }
      named_bar_sync(bar_id, 128);
      if (row_in_tile < 16) {
        const int j = row_in_tile;
        const int tok = tok0 + j;
        if (tok < e.M) {
          LmPart p;
          p.mx = red_f[64 + j];
          p.se = ((red_f[j] + red_f[16 + j]) + red_f[32 + j]) + red_f[48 + j];
          p.idx = red_i[64 + j];
          p.pad = 0;
          e.lm_part[static_cast<size_t>(tok) * e.lm_tiles + row_tile] = p;
        }
      }
      named_bar_sync(bar_id, 128);
    } break;
  }
}

// RoPE position of row r (0-based in its sequence's forward) relative to the first row's
// position.  Plain forwards: r.  Quadratic self-speculation (quad_k = k): rows 0..k verify
// [x_n, d_1..d_k] at offsets 0..k; row k+1+a*k+j (pre-draft block a = 0..k, slot j = 0..k-1)
// sits at offset a+1+j, while its K/V goes to slot r like every row.
NLD_DEV int rope_offset(int r, int quad_k) {
  if (quad_k <= 0 || r <= quad_k) return r;
  const int q = r - quad_k - 1;
  return q / quad_k + 1 + q % quad_k;
}

// Per-column data of a tile of n token columns starting at tok0 (see epi_chunk): 1/rms from
// the RMSNorm statistics when `norm` (lane l of a warp sums tiles l, l+32, ... of 8 tokens at
// once, then a shuffle reduction finishes each token), and for the QKV epilogue the KV slot, its
// page and the RoPE position of each token.  nthr threads (a multiple of 32) share the work.
NLD_DEV void compute_tile_meta(const EpiArgs& e, int tok0, int n, bool norm, float* s_inv,
                               int* s_pos, int* s_pg, int* s_rpos, int et, int nthr) {
  const int nw = nthr >> 5, w = et >> 5, lane = et & 31;
  if (norm) {
    for (int c0 = w; c0 < n; c0 += nw * 8) {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        acc[q] = 0.f;
        const int c = c0 + q * nw;
        const int tok = tok0 + c;
        if (c < n && tok < e.M)
          for (int t = lane; t < e.ssq_tiles; t += 32)
            acc[q] += __ldg(&e.ssq_in[static_cast<size_t>(t) * e.ssq_ld + tok]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float v = acc[q];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        const int c = c0 + q * nw;
        if (lane == 0 && c < n) s_inv[c] = (tok0 + c < e.M) ? rsqrtf(v * e.inv_d + e.eps) : 0.f;
      }
    }
  }
  if (e.kind == EPI_QKV) {
    for (int c = et; c < n; c += nthr) {
      const int tok = tok0 + c;
      int pos = -1, pg = 0, rpos = -1;
      if (tok < e.M) {
        const int b = tok / e.m;
        const int len = __ldg(&e.lens[b]);
        pos = len + (tok - b * e.m);
        rpos = len + rope_offset(tok - b * e.m, e.quad_k);
        if (pos >= e.kv_cap || pos < 0) {
          set_err(e.err, NLD_DEVERR_KV_OVERFLOW);
          pos = rpos = -1;
        } else {
          pg = __ldg(&e.page_table[b * e.pps + (pos >> 6)]);
        }
      }
      s_pos[c] = pos;
      s_pg[c] = pg;
      s_rpos[c] = rpos;
    }
  }
}

}  // namespace nld
