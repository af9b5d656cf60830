// The router's backward with the top-K selection held fixed.
//
// "Two upstream innovations of MoE: Routing-Free and OmniMoE", section 1.1 (Router ->
// Softmax -> TopK) and "How AI chips support MoE", chapter 4, section 4.2 (the gate is the
// linear map x W_r + bias), read backwards. With d_w = dL/dw[t, k] (from the expert half's
// backward) and s_t = sum_k w[t, k] d_w[t, k]:
//   renormalised top-K softmax: dL/dl[t, e] = w[t, k] (d_w[t, k] - s_t) if e = id[t, k],
//                               0 for an expert that was not selected;
//   plain softmax over all E:   dL/dl[t, e] = p[t, e] (g[t, e] - s_t), g = d_w at the
//                               selected experts, 0 elsewhere;
//   d_W_r = x^T dL/dl, d_bias = sum_t dL/dl[t, :], and the router's term of the input
//   gradient dL/dl W_r^T, added to d_x.
// Three kernels: one warp per token for dL/dl (the K selections are held one per lane and
// broadcast by shuffles; a warp max and sum give the plain softmax); d_W_r and d_bias by
// CTAs that own 32 columns of W_r and EC experts and sum over all tokens in a fixed order
// (sixteen token groups, then the groups in order: deterministic); the input-gradient term
// by CTAs that own 64 columns of d with that slice of W_r in shared memory, 8 threads per
// token row slice, fp32 sums added to the bf16 d_x. Routers with more than 16 experts run
// the last two on the tensor cores (route_bwd_tc.cu) where E % 8 == 0 and the operands are
// 16-byte aligned, else in the register-tiled forms below.
#include <math.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) router_dlogits_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ topk_w,
    const float* __restrict__ d_w, const float* __restrict__ logits, int T, int E, int K,
    int renorm, float* __restrict__ d_logits) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int warps = (int)(gridDim.x * (blockDim.x >> 5));
  for (int t = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)); t < T; t += warps) {
    int id = -1;
    float w = 0.f, g = 0.f;
    if (lane < K) {
      id = ids[(size_t)t * K + lane];
      w = topk_w[(size_t)t * K + lane];
      g = d_w[(size_t)t * K + lane];
    }
    float s = w * g;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // plain softmax: p over all E (max and sum over the warp)
    float m = -INFINITY, den = 0.f;
    if (!renorm) {
      for (int e = lane; e < E; e += 32) m = fmaxf(m, logits[(size_t)t * E + e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      for (int e = lane; e < E; e += 32) den += expf(logits[(size_t)t * E + e] - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    for (int e0 = 0; e0 < E; e0 += 32) {  // warp-uniform
      const int e = e0 + lane;
      float ge = 0.f, we = 0.f;
      bool sel = false;
      for (int k = 0; k < K; ++k) {
        const int ik = __shfl_sync(0xffffffffu, id, k);
        const float wk = __shfl_sync(0xffffffffu, w, k);
        const float gk = __shfl_sync(0xffffffffu, g, k);
        if (ik == e) {
          sel = true;
          we = wk;
          ge = gk;
        }
      }
      if (e < E) {
        float v;
        if (renorm) v = sel ? we * (ge - s) : 0.f;
        else v = expf(logits[(size_t)t * E + e] - m) / den * (ge - s);
        d_logits[(size_t)t * E + e] = v;
      }
    }
  }
}

// d_W_r[j, e] = sum_t x[t, j] dl[t, e]; d_bias[e] = sum_t dl[t, e] (CTAs of column block 0).
// CTA: 32 columns of x (one per lane) x EC experts; warp w of the 16 sums the tokens
// t = w (mod 16), eight tokens' loads issued before any is used.
constexpr int kDwrWarps = 16;
constexpr int kDwrUnroll = 8;

template <int EC>
__global__ void __launch_bounds__(kDwrWarps * 32) router_dwr_kernel(
    const bf16* __restrict__ x, const float* __restrict__ dl, int T, int d, int E,
    float* __restrict__ d_w_r, float* __restrict__ d_bias) {
  __shared__ float red[kDwrWarps][32][EC + 1];
  __shared__ float redb[kDwrWarps][EC + 1];
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = blockIdx.x * 32 + lane;  // column of x / row of W_r
  const int e0 = blockIdx.y * EC;
  const bool bias_cta = blockIdx.x == 0 && d_bias != nullptr;
  const bool ecol = lane < EC && e0 + lane < E;
  float acc[EC], accb[EC];
#pragma unroll
  for (int q = 0; q < EC; ++q) acc[q] = accb[q] = 0.f;
  for (int t0 = warp; t0 < T; t0 += kDwrWarps * kDwrUnroll) {
    float xv[kDwrUnroll], dv[kDwrUnroll];
#pragma unroll
    for (int u = 0; u < kDwrUnroll; ++u) {
      const int t = t0 + u * kDwrWarps;
      xv[u] = (t < T && j < d) ? __bfloat162float(x[(size_t)t * d + j]) : 0.f;
      dv[u] = (t < T && ecol) ? dl[(size_t)t * E + e0 + lane] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kDwrUnroll; ++u)
#pragma unroll
      for (int q = 0; q < EC; ++q) {
        const float dq = __shfl_sync(0xffffffffu, dv[u], q);
        acc[q] = fmaf(xv[u], dq, acc[q]);
        if (bias_cta) accb[q] += dq;
      }
  }
#pragma unroll
  for (int q = 0; q < EC; ++q) red[warp][lane][q] = acc[q];
  if (bias_cta && lane == 0)
#pragma unroll
    for (int q = 0; q < EC; ++q) redb[warp][q] = accb[q];
  __syncthreads();
  for (int i = threadIdx.x; i < 32 * EC; i += kDwrWarps * 32) {
    const int c = i / EC, q = i % EC;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDwrWarps; ++w) v += red[w][c][q];  // token groups in order
    const int jj = blockIdx.x * 32 + c, e = e0 + q;
    if (jj < d && e < E) d_w_r[(size_t)jj * E + e] = v;
  }
  if (bias_cta && threadIdx.x < EC && e0 + (int)threadIdx.x < E) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDwrWarps; ++w) v += redb[w][threadIdx.x];
    d_bias[e0 + threadIdx.x] = v;
  }
}

// d_x[t, j] += sum_e dl[t, e] W_r[j, e]. CTA: 64 columns of d (its W_r slice in shared
// memory, fp32, expert-major), 8 threads per token row slice (8 columns each, one 16-byte
// vector of d_x).
__global__ void __launch_bounds__(256) router_dx_kernel(const bf16* __restrict__ w_r,
                                                        const float* __restrict__ dl, int T,
                                                        int d, int E, int tokens_per_cta,
                                                        bf16* __restrict__ d_x) {
  extern __shared__ float wsl[];  // [E][64]: expert-major, a thread's 8 columns contiguous
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int j0 = blockIdx.x * 64;
  for (int i = threadIdx.x; i < 64 * E; i += 256) {
    const int r = i / E, e = i % E;
    wsl[e * 64 + r] = (j0 + r < d) ? __bfloat162float(w_r[(size_t)(j0 + r) * E + e]) : 0.f;
  }
  __syncthreads();
  const int sub = threadIdx.x & 7;   // 8 columns [j0 + 8 sub, +8)
  const int row = threadIdx.x >> 3;  // 32 tokens per pass
  const int t_begin = blockIdx.y * tokens_per_cta;
  const int t_end = min(T, t_begin + tokens_per_cta);
  const int jj = j0 + sub * 8;
  if (jj >= d) return;
  for (int t = t_begin + row; t < t_end; t += 32) {
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.f;
    const float* dlt = dl + (size_t)t * E;
    uint4* px = reinterpret_cast<uint4*>(d_x + (size_t)t * d + jj);
    const uint4 old = *px;  // issued before the sums that follow
    for (int ec = 0; ec < E; ec += 8) {  // eight of the token's d_logits loaded together
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ec + u < E ? dlt[ec + u] : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (ec + u >= E) continue;
        const float4 w0 = *reinterpret_cast<const float4*>(wsl + (ec + u) * 64 + sub * 8);
        const float4 w1 = *reinterpret_cast<const float4*>(wsl + (ec + u) * 64 + sub * 8 + 4);
        acc[0] = fmaf(v[u], w0.x, acc[0]);
        acc[1] = fmaf(v[u], w0.y, acc[1]);
        acc[2] = fmaf(v[u], w0.z, acc[2]);
        acc[3] = fmaf(v[u], w0.w, acc[3]);
        acc[4] = fmaf(v[u], w1.x, acc[4]);
        acc[5] = fmaf(v[u], w1.y, acc[5]);
        acc[6] = fmaf(v[u], w1.z, acc[6]);
        acc[7] = fmaf(v[u], w1.w, acc[7]);
      }
    }
    float cur[8];
    unpack16(old, cur, bf16());
#pragma unroll
    for (int c = 0; c < 8; ++c) cur[c] += acc[c];
    *px = pack16(cur, bf16());
  }
}

// ---- wide routers (E > 16): register-tiled CUDA-core GEMMs, fp32 throughout.
// d_W_r = x^T dl: a 64 (columns of x) x 64 (experts) tile per cluster of 4 CTAs; each CTA
// sums a quarter of the tokens (chunks of 32 staged in shared memory, a 4 x 4 register tile
// per thread), then CTA rank 0 adds the four partial tiles in rank order through
// distributed shared memory (deterministic, no global scratch). d_bias comes from the
// column-tile-0 clusters the same way.
constexpr int kWt = 64, kWk = 32, kWsplit = 4;

__global__ void __launch_bounds__(256) router_dwr_tiled_kernel(const bf16* __restrict__ x,
                                                               const float* __restrict__ dl,
                                                               int T, int d, int E,
                                                               float* __restrict__ d_w_r,
                                                               float* __restrict__ d_bias) {
  __shared__ __align__(16) float xs[kWk][kWt];  // [token][column]
  __shared__ __align__(16) float ds[kWk][kWt];  // [token][expert]
  __shared__ __align__(16) float part[kWt][kWt + 1];
  __shared__ float partb[kWt];
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const uint32_t rank = ptx::cluster_rank();
  const int tile = blockIdx.x / kWsplit;
  const int e_tiles = (E + kWt - 1) / kWt;
  const int jt = tile / e_tiles, et = tile % e_tiles;
  const int j0 = jt * kWt, e0 = et * kWt;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 each
  const bool bias = d_bias != nullptr && jt == 0;
  const int per = (T + kWsplit - 1) / kWsplit;
  const int t_begin = (int)rank * per, t_end = min(T, t_begin + per);
  float acc[4][4], accb[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    accb[i] = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
  }
  // loaders: x chunk 32 x 64 bf16 = one 8-element vector per thread; dl chunk 32 x 64 fp32 =
  // eight values per thread; the next chunk's loads are issued before this chunk's sums
  const int lr = threadIdx.x >> 3, lc = (threadIdx.x & 7) * 8;
  uint4 xr = make_uint4(0, 0, 0, 0);
  float dr[8];
  auto load = [&](int t0) {
    const int t = t0 + lr;
    xr = t < t_end ? *reinterpret_cast<const uint4*>(x + (size_t)t * d + j0 + lc)
                   : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int e = e0 + lc + c;
      dr[c] = (t < t_end && e < E) ? dl[(size_t)t * E + e] : 0.f;
    }
  };
  if (t_begin < t_end) load(t_begin);
  for (int t0 = t_begin; t0 < t_end; t0 += kWk) {
    {
      float f[8];
      unpack16(xr, f, bf16());
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        xs[lr][lc + c] = f[c];
        ds[lr][lc + c] = dr[c];
      }
    }
    __syncthreads();
    if (t0 + kWk < t_end) load(t0 + kWk);
#pragma unroll 8
    for (int kk = 0; kk < kWk; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ds[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
      if (bias && ty == 0)
#pragma unroll
        for (int q = 0; q < 4; ++q) accb[q] += bv[q];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int q = 0; q < 4; ++q) part[ty * 4 + i][tx * 4 + q] = acc[i][q];
  if (bias && ty == 0)
#pragma unroll
    for (int q = 0; q < 4; ++q) partb[tx * 4 + q] = accb[q];
  ptx::cluster_sync();  // every rank's partial tile is in its shared memory
  if (rank == 0) {
    for (int i = threadIdx.x; i < kWt * kWt; i += 256) {
      const int r = i / kWt, c = i % kWt;
      float v = part[r][c];
      for (uint32_t q = 1; q < kWsplit; ++q)  // rank order
        v += ptx::ld_dsmem_f32(ptx::map_rank(ptx::saddr(&part[r][c]), q));
      const int j = j0 + r, e = e0 + c;
      if (j < d && e < E) d_w_r[(size_t)j * E + e] = v;
    }
    if (bias && threadIdx.x < kWt) {
      float v = partb[threadIdx.x];
      for (uint32_t q = 1; q < kWsplit; ++q)
        v += ptx::ld_dsmem_f32(ptx::map_rank(ptx::saddr(&partb[threadIdx.x]), q));
      const int e = e0 + (int)threadIdx.x;
      if (e < E) d_bias[e] = v;
    }
  }
  ptx::cluster_sync();  // the peers' tiles have been read; they may exit
}

// d_x[t, j] += sum_e dl[t, e] W_r[j, e]: a CTA owns 64 tokens and kDxCols columns. Its
// tokens' dl rows are staged once in shared memory (expert-major), then each 64-column tile
// sums over the experts in chunks of 32 (the W_r chunk staged expert-major, the next
// chunk's loads issued before this chunk's sums), a 4 x 4 register tile per thread; fp32
// sums added to the bf16 d_x.
constexpr int kDxCols = 512;

__global__ void __launch_bounds__(256) router_dx_tiled_kernel(const bf16* __restrict__ w_r,
                                                              const float* __restrict__ dl,
                                                              int T, int d, int E, int Ep,
                                                              bf16* __restrict__ d_x) {
  extern __shared__ __align__(16) float dsm[];
  float* ls = dsm;               // [Ep][64]: expert-major dl of the CTA's tokens
  float* ws = dsm + Ep * kWt;    // [32][64]: expert-major W_r chunk
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  const int t0 = blockIdx.x * kWt;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  for (int i = threadIdx.x; i < kWt * Ep; i += 256) {
    const int r = i / Ep, e = i % Ep;  // consecutive threads: consecutive experts of a token
    ls[e * kWt + r] = (t0 + r < T && e < E) ? dl[(size_t)(t0 + r) * E + e] : 0.f;
  }
  const int lr = threadIdx.x >> 2, lc = (threadIdx.x & 3) * 8;
  float wv[8];
  for (int j0 = blockIdx.y * kDxCols; j0 < min(d, (int)(blockIdx.y + 1) * kDxCols); j0 += kWt) {
    auto load = [&](int k0) {
      const int j = j0 + lr;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = k0 + lc + u;
        wv[u] = (j < d && e < E) ? __bfloat162float(w_r[(size_t)j * E + e]) : 0.f;
      }
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
    load(0);
    for (int k0 = 0; k0 < E; k0 += kWk) {
      __syncthreads();  // the previous chunk's sums are done with ws (and ls is complete)
#pragma unroll
      for (int u = 0; u < 8; ++u) ws[(lc + u) * kWt + lr] = wv[u];
      __syncthreads();
      if (k0 + kWk < E) load(k0 + kWk);
#pragma unroll 8
      for (int kk = 0; kk < kWk; ++kk) {
        const float4 a = *reinterpret_cast<const float4*>(&ls[(k0 + kk) * kWt + ty * 4]);
        const float4 b = *reinterpret_cast<const float4*>(&ws[kk * kWt + tx * 4]);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(av[i], bv[q], acc[i][q]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + ty * 4 + i, j = j0 + tx * 4;
      if (t >= T || j >= d) continue;
      uint2* px = reinterpret_cast<uint2*>(d_x + (size_t)t * d + j);
      const uint2 old = *px;
      const float c0 = __uint_as_float(old.x << 16) + acc[i][0];
      const float c1 = __uint_as_float(old.x & 0xffff0000u) + acc[i][1];
      const float c2 = __uint_as_float(old.y << 16) + acc[i][2];
      const float c3 = __uint_as_float(old.y & 0xffff0000u) + acc[i][3];
      *px = make_uint2(pack_bf16x2(c0, c1), pack_bf16x2(c2, c3));
    }
  }
}

}  // namespace

// route_bwd_tc.cu: the tensor-core forms of d_W_r (with d_bias) and of the d_x term; they
// set *used = false for the shapes and alignments they do not take.
moe_status launch_router_dwr_tc(const moe_shape& s, const void* x, const float* d_logits,
                                float* d_w_r, float* d_bias, cudaStream_t st, bool* used);
moe_status launch_router_dx_tc(const moe_shape& s, const void* w_r, const float* d_logits,
                               void* d_x, cudaStream_t st, bool* used);

moe_status launch_router_backward(const moe_shape& s, const void* x, const void* w_r,
                                  const float* logits, const int32_t* ids, const float* topk_w,
                                  const float* d_w, float* d_logits, float* d_w_r,
                                  float* d_bias, void* d_x, cudaStream_t st) {
  const int T = s.T, d = s.d, E = s.E, K = s.K;
  moe_status r;
  {
    long long blocks = ((long long)T + 7) / 8;
    if (blocks > (long long)sm_count() * 8) blocks = (long long)sm_count() * 8;
    launch_begin(K_ROUTER_DLOGITS, st);
    launch_kernel(router_dlogits_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, ids, topk_w,
                  d_w, logits, T, E, K, s.renormalize, d_logits);
    if ((r = launch_end(K_ROUTER_DLOGITS, st)) != MOE_OK) return r;
  }
  bool tc = false;
  if (E > 16 && (r = launch_router_dwr_tc(s, x, d_logits, d_w_r, d_bias, st, &tc)) != MOE_OK)
    return r;
  if (E > 16 && !tc) {  // the CUDA-core forms for the other wide routers
    const int tiles = ((d + kWt - 1) / kWt) * ((E + kWt - 1) / kWt);
    launch_begin(K_ROUTER_DWR, st);
    launch_kernel(router_dwr_tiled_kernel, dim3((unsigned)(tiles * kWsplit)), dim3(256), 0, st,
                  (unsigned)kWsplit, (const bf16*)x, (const float*)d_logits, T, d, E, d_w_r,
                  d_bias);
    if ((r = launch_end(K_ROUTER_DWR, st)) != MOE_OK) return r;
  } else if (E <= 16) {
    const int EC = E <= 8 ? 8 : 16;
    const dim3 grid((unsigned)((d + 31) / 32), (unsigned)((E + EC - 1) / EC));
    const dim3 block(kDwrWarps * 32);
    launch_begin(K_ROUTER_DWR, st);
    if (EC == 8)
      launch_kernel(router_dwr_kernel<8>, grid, block, 0, st, 1, (const bf16*)x,
                    (const float*)d_logits, T, d, E, d_w_r, d_bias);
    else
      launch_kernel(router_dwr_kernel<16>, grid, block, 0, st, 1, (const bf16*)x,
                    (const float*)d_logits, T, d, E, d_w_r, d_bias);
    if ((r = launch_end(K_ROUTER_DWR, st)) != MOE_OK) return r;
  }
  tc = false;
  if (d_x != nullptr && E > 16 &&
      (r = launch_router_dx_tc(s, w_r, d_logits, d_x, st, &tc)) != MOE_OK)
    return r;
  if (d_x != nullptr && E > 16 && !tc) {
    const int Ep = (E + kWk - 1) / kWk * kWk;  // experts padded to whole chunks
    const int smem = (Ep + kWk) * kWt * (int)sizeof(float);
    if (cudaFuncSetAttribute(router_dx_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_begin(K_ROUTER_DX, st);
    launch_kernel(router_dx_tiled_kernel,
                  dim3((unsigned)((T + kWt - 1) / kWt), (unsigned)((d + kDxCols - 1) / kDxCols)),
                  dim3(256), (size_t)smem, st, 1, (const bf16*)w_r, (const float*)d_logits, T, d,
                  E, Ep, (bf16*)d_x);
    if ((r = launch_end(K_ROUTER_DX, st)) != MOE_OK) return r;
  } else if (d_x != nullptr && E <= 16) {
    const int smem = 64 * E * (int)sizeof(float);
    if (cudaFuncSetAttribute(router_dx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int col_blocks = (d + 63) / 64;
    int tok_blocks = (sm_count() * 4 + col_blocks - 1) / col_blocks;
    if (tok_blocks < 1) tok_blocks = 1;
    const int tpc = (T + tok_blocks - 1) / tok_blocks;
    tok_blocks = (T + tpc - 1) / tpc;
    launch_begin(K_ROUTER_DX, st);
    launch_kernel(router_dx_kernel, dim3((unsigned)col_blocks, (unsigned)tok_blocks), dim3(256),
                  (size_t)smem, st, 1, (const bf16*)w_r, (const float*)d_logits, T, d, E, tpc,
                  (bf16*)d_x);
    if ((r = launch_end(K_ROUTER_DX, st)) != MOE_OK) return r;
  }
  return MOE_OK;
}

}  // namespace moe
