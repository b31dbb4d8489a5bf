// fp32 projection GEMM on the CUDA cores for the fp32 configuration (tf32 tensor-core inputs
// would carry ~1e-3 relative error, above the fp32 tolerance).  One CTA = 128 weight rows x 16
// tokens; W and X tiles are staged through shared memory; each thread accumulates one row in
// fp32 and then runs the same fused epilogue as the tensor-core kernel.
#include "common.cuh"
#include "epilogue.cuh"

namespace nld {

__global__ void __launch_bounds__(128)
    gemm_simt_kernel(const float* __restrict__ W, const float* __restrict__ X, int n_rows, int K,
                     int M, const EpiArgs e) {
  __shared__ float Ws[kTileRows][33];
  __shared__ float Xs[16][33];
  __shared__ float s_inv[16];
  __shared__ int s_pos[16];
  __shared__ int s_pg[16];
  __shared__ int s_rpos[16];
  __shared__ float red_f[96];
  __shared__ int red_i[96];
  pdl_wait();
  pdl_launch_dependents();
  const int rt = blockIdx.x;
  const int tok0 = blockIdx.y * 16;
  const int tid = threadIdx.x;
  compute_tile_meta(e, tok0, 16, e.kind != EPI_RESID, s_inv, s_pos, s_pg, s_rpos, tid, 128);
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int idx = tid; idx < kTileRows * 32; idx += 128) {
      const int r = idx >> 5, c = idx & 31;
      const int gr = rt * kTileRows + r;
      Ws[r][c] = (gr < n_rows) ? W[static_cast<size_t>(gr) * K + k0 + c] : 0.f;
    }
    for (int idx = tid; idx < 16 * 32; idx += 128) {
      const int t = idx >> 5, c = idx & 31;
      Xs[t][c] = (tok0 + t < M) ? X[static_cast<size_t>(tok0 + t) * K + k0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float w = Ws[tid][kk];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = fmaf(w, Xs[j][kk], acc[j]);
    }
    __syncthreads();
  }
  EpiPre pre;
  epi_preload(e, rt, tid, tok0, s_rpos, 0, pre);
  epi_chunk<float>(e, rt, tid, tid & 31, tid >> 5, tok0, s_inv, s_pos, s_pg, 0, acc, pre, red_f, red_i, 1);
}

cudaError_t launch_gemm_simt(cudaStream_t st, const float* W, const float* X, int n_rows, int K,
                             int M, const EpiArgs& e, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((n_rows + kTileRows - 1) / kTileRows, (M + 15) / 16);
  cfg.blockDim = dim3(128);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, gemm_simt_kernel, W, X, n_rows, K, M, e);
}

}  // namespace nld
