// Weighted combine back to token order.
//
// SonicMoE explainer (gitcode.csdn.net), section 3 item 6: scatter/combine back to the
// token-major layout; section 6.1: the aggregation kernel fuses the scatter and the sum.
//   out[t] = sum_{k, assign_to_perm[t*K+k] >= 0} topk_w[t,k] * y_perm[assign_to_perm[t*K+k]]
// fp32 accumulation in k order (deterministic); dropped slots add nothing.
//
// HBM-bound. One thread per (token, 16-byte column vector): the K expert rows are read
// with independent 128-bit loads (K loads in flight per thread), consecutive threads take
// consecutive vectors of one row, so every warp access is 512 contiguous bytes.
#include "common.cuh"

namespace moe {

namespace {

template <typename Tv>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ a2p,
                                                      const float* __restrict__ topk_w, int T,
                                                      int K, int vec_per_row, long long n_rows,
                                                      uint4* __restrict__ out, unsigned* status) {
  constexpr int V = Vec16<Tv>::N;
  const long long total = (long long)T * vec_per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / vec_per_row;
    const int v = (int)(i - t * vec_per_row);
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 4) {  // up to 4 rows in flight
      uint4 u[4];
      float w[4];
      bool ok[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = k0 + j;
        ok[j] = false;
        if (k < K) {
          const long long p = a2p[t * K + k];
          if (p >= n_rows) report(status, MOE_ERR_DEVICE_INDEX);
          if (p >= 0 && p < n_rows) {
            ok[j] = true;
            w[j] = topk_w[t * K + k];
            u[j] = y_perm[p * vec_per_row + v];
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!ok[j]) continue;
        float f[V];
        unpack16(u[j], f, Tv());
#pragma unroll
        for (int q = 0; q < V; ++q) acc[q] = fmaf(w[j], f[q], acc[q]);
      }
    }
    out[i] = pack16(acc, Tv());
  }
}

}  // namespace

moe_status launch_combine(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                          const float* topk_w, void* out, cudaStream_t st) {
  const int elem = (s.dtype == MOE_BF16) ? 2 : 4;
  const int vec_per_row = s.d * elem / 16;
  const long long total = (long long)s.T * vec_per_row;
  if (total == 0) return MOE_OK;
  long long blocks = (total + 255) / 256;
  const long long cap_blocks = (long long)sm_count() * 8;
  if (blocks > cap_blocks) blocks = cap_blocks;
  const long long n_rows = (long long)s.T * s.K;
  launch_begin(K_COMBINE, st);
  if (s.dtype == MOE_BF16)
    combine_kernel<bf16><<<(int)blocks, 256, 0, st>>>((const uint4*)y_perm, a2p, topk_w, s.T, s.K,
                                                      vec_per_row, n_rows, (uint4*)out,
                                                      device_status_ptr());
  else
    combine_kernel<float><<<(int)blocks, 256, 0, st>>>((const uint4*)y_perm, a2p, topk_w, s.T, s.K,
                                                       vec_per_row, n_rows, (uint4*)out,
                                                       device_status_ptr());
  return launch_end(K_COMBINE, st);
}

}  // namespace moe
