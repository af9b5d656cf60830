// The router's two backward contractions on the tensor cores (tcgen05), for routers of more
// than 16 experts:
//   d_W_r = x^T dL/dl         ([d, E] fp32: x [T, d] bf16, dL/dl [T, E] fp32)
//   d_x  += dL/dl W_r^T       ([T, d] bf16: W_r [d, E] bf16)
// ("Two upstream innovations of MoE: Routing-Free and OmniMoE", section 1.1, and "How AI
// chips support MoE", chapter 4, section 4.2: the gate is the linear map x W_r + bias; these
// are its two gradients.) d_bias, the column sums of dL/dl, is formed beside d_W_r in fp32.
//
// Precision. The tensor cores multiply bf16 pairs; dL/dl is fp32. Each of its values v is
// split into two bf16 terms, hi = bf16(v) and lo = bf16(v - hi) (v - hi is exact in fp32),
// and every product is issued twice, hi then lo, into the same fp32 accumulator. Both
// roundings are to nearest with 8 significant bits, so |v - hi - lo| <= 2^-16 |v| and the
// sums keep the fp32 operand's accuracy: the operand-splitting of Markidis et al., "NVIDIA
// Tensor Core Programmability, Performance & Precision" (2018), with bf16 terms. x and W_r
// are bf16 already, so their products with hi and lo are exact in fp32.
//
// d_W_r (router_dwr_tc_kernel): D[j, e] = sum_t x[t, j] dL/dl[t, e] for 128 columns j of x
// (the MMA's M) and one chunk of up to 64 experts (N: the chunk's experts rounded up to 32);
// K = tokens in blocks of 64. A = x[t, j] tiles by TMA, MN-major (two [64 t][64 j]
// 128-byte-swizzled chunks); B = the chunk's dL/dl values as hi / lo terms, converted by eight
// warps (one float4 per thread and row, so a warp reads two whole 256-byte row segments) and
// written in the layout TMA would give a [64 t][64 e] box (MN-major, 128-byte swizzle). The
// tokens are split over the S CTAs of a cluster (contiguous ranges of whole blocks); after
// the last MMA each CTA copies its partial tile to shared memory and, after a cluster
// barrier, CTA q adds the S partials of rows [q 128/S, (q+1) 128/S) in rank order through
// distributed shared memory (the same fp32 sums in the same order on every run). The
// converters also add up their fp32 values per expert in token order; d_bias is the
// cluster's rank-ordered sum of those. Three 32 KB stages, two CTAs per SM. Roles (320
// threads): warp 0 issues the x loads, warp 1 the MMAs, warps 2-9 convert; warps 2-5 read
// the accumulator (warp w may read TMEM lanes 32 (w % 4) ...).
//
// d_x: D[t, j] = sum_e dL/dl[t, e] W_r[j, e], 128 tokens on M and 128 columns of d on N,
// K = experts (at most 256: one shot per tile). A = the tile's dL/dl rows as hi and lo terms
// (K-major, converted by all threads, one float4 each), B = W_r rows by TMA (K-major: W_r is
// [d, E] with E innermost); the sums are added to the bf16 d_x and rounded once, as the
// CUDA-core form does. Two kernels:
//  - E <= 128, router_dx_tc_stream_kernel: one CTA per token tile converts A once and
//    streams the column tiles, d_x moving by TMA through a 3-stage ring (described below);
//  - E > 128, router_dx_tc_kernel: one CTA per 128 x 128 tile (A and B leave no room for the
//    ring); the tile's d_x values are loaded at the start (whole 128-byte row segments per 8
//    threads) and after the MMAs the sums go through shared memory in two 64-column halves,
//    so that the read-add-store of d_x runs on that row-contiguous pattern.
//
// Every mbarrier wait is bounded: on expiry the status word records MOE_ERR_TIMEOUT, the
// abort flag makes the CTA's other waits give up, nothing is stored, and the TMEM and the
// cluster barriers are still released and passed.
#include <mutex>

#include "common.cuh"
#include "ffn_args.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace ptx;

constexpr int kChunk = 64 * 128;  // 8 KB: [64 rows][64 bf16], one 128-byte swizzle span a row

// Byte offset of the 8-byte half h of 16-byte unit u (of 8) in row r of a 128-byte-swizzled
// span of 8-row groups: the unit index is XORed with the row's index inside its group.
__device__ __forceinline__ int sw128(int r, int u, int h) {
  return r * 128 + ((u ^ (r & 7)) << 4) + (h << 3);
}

// Four fp32 values as two bf16 pairs hi and lo with v = hi + lo + (|error| <= 2^-16 |v|).
__device__ __forceinline__ void split4(const float4& v, uint2& hi, uint2& lo) {
  hi.x = pack_bf16x2(v.x, v.y);
  hi.y = pack_bf16x2(v.z, v.w);
  lo.x = pack_bf16x2(v.x - __uint_as_float(hi.x << 16), v.y - __uint_as_float(hi.x & 0xffff0000u));
  lo.y = pack_bf16x2(v.z - __uint_as_float(hi.y << 16), v.w - __uint_as_float(hi.y & 0xffff0000u));
}

// Four consecutive dL/dl values of token t from expert e (E % 4 == 0: all in or all out).
__device__ __forceinline__ float4 load4(const float* __restrict__ dl, int t, int T, int e, int E) {
  return (t < T && e < E) ? __ldg(reinterpret_cast<const float4*>(dl + (size_t)t * E + e))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// ------------------------------------------------------------------ d_W_r and d_bias
constexpr int kWrThreads = 320;
constexpr int kWrConv = 256;  // converter threads (warps 2-9)
constexpr int kWrStages = 3;
constexpr int kWrStage = 2 * kChunk + 2 * kChunk;  // x chunk pair + hi + lo: 32 KB
constexpr int kWrTmemCols = 64;
constexpr int kWrPs = 64 + 4;  // row stride (floats) of the partial tile in shared memory
constexpr int kWrRows = 4;     // rows of a block per converter thread (16 threads a row)
constexpr int kWrExtra = (kWrConv * 4 + 64) * 4 + (2 * kWrStages + 1) * 8 + 16;
constexpr int kWrSmem = 1024 + kWrStages * kWrStage + kWrExtra;
static_assert(128 * kWrPs * 4 <= kWrStages * kWrStage, "the partial tile fits the ring");

struct DwrArgs {
  const float* dl;
  float* d_w_r;
  float* d_bias;
  int T, d, E;
  int nchunks;   // 64-expert chunks: ceil(E / 64); cluster c takes chunk c % nchunks
  int S;         // CTAs of a cluster splitting the tokens
  int kb_total;  // blocks of 64 tokens: ceil(T / 64)
  unsigned* status;
  unsigned long long limit_ns;
};

__global__ void __launch_bounds__(kWrThreads, 2)
    router_dwr_tc_kernel(const __grid_constant__ CUtensorMap tmX, const DwrArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = align1024(smem_raw);
  float* bias_part = (float*)(ring + kWrStages * kWrStage);  // [256 converters][4]
  float* cta_bias = bias_part + kWrConv * 4;                 // [64]
  uint64_t* full = (uint64_t*)(cta_bias + 64);
  uint64_t* empty = full + kWrStages;
  uint64_t* accf = empty + kWrStages;
  uint32_t* tmem_slot = (uint32_t*)(accf + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = g.S;
  const uint32_t rank = cluster_rank();  // 0 without a cluster
  const int cid = (int)cluster_id_x();
  const int chunk = cid % g.nchunks, mtile = cid / g.nchunks;
  const int j0 = mtile * 128, e0 = 64 * chunk;
  const int Ec = min(64, g.E - e0);          // this chunk's experts (a multiple of 8)
  const int NE = (Ec + 31) / 32 * 32;        // the MMA's N
  const int kb0 = (int)((long long)rank * g.kb_total / S);
  const int nkb = (int)((long long)(rank + 1) * g.kb_total / S) - kb0;

  if (tid == 32) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmX) : "memory");
  if (tid == 0) {
    for (int s = 0; s < kWrStages; ++s) {
      mbar_init(saddr(&full[s]), 1 + kWrConv);  // the x loads' expect_tx + every converter
      mbar_init(saddr(&empty[s]), 1);
    }
    mbar_init(saddr(accf), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc<1>(saddr(tmem_slot), kWrTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the previous kernel in the stream has completed (it wrote dL/dl)
  pdl_trigger();

  if (warp == 0) {
    // ---- x producer: both 64-column chunks of the tile for each block of 64 tokens
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (lane == 0) {
        const uint32_t fb = saddr(&full[stage]);
        const uint32_t a = saddr(ring + stage * kWrStage);
        const int tk = (kb0 + i) * 64;
        mbar_expect_tx(fb, 2 * kChunk);
        tma_load_2d(a, &tmX, j0, tk, fb);
        tma_load_2d(a + kChunk, &tmX, j0 + 64, tk, fb);
      }
      __syncwarp();
      if (++stage == kWrStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue: per block, 4 steps of 16 tokens, each as hi then lo
    // A (MN-major): 64-column chunks 8 KB apart, 8-row groups 1 KB apart, a step = 16 rows.
    // B (MN-major): one 64-expert chunk, the same row geometry.
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           ((uint32_t)(NE >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&full[stage]), phase, abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a = saddr(ring + stage * kWrStage);
        const uint32_t bh = a + 2 * kChunk, bl = bh + kChunk;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t ad = desc_sw128(a + s * 2048, kChunk, 1024);
          tc_mma<1>(tmem, ad, desc_sw128(bh + s * 2048, kChunk, 1024), idesc,
                    (i | s) != 0 ? 1u : 0u);
          tc_mma<1>(tmem, ad, desc_sw128(bl + s * 2048, kChunk, 1024), idesc, 1u);
        }
        tc_commit<1>(saddr(&empty[stage]));
      }
      __syncwarp();
      if (++stage == kWrStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0) tc_commit<1>(saddr(accf));  // arrives at once if nothing was issued
    __syncwarp();
  } else {
    // ---- converters: thread c owns experts e0 + 4 q .. + 3 (q = c % 16) of the rows
    // rl, rl + 16, rl + 32, rl + 48 (rl = c / 16) of every block
    const int c = tid - 64;
    const int q = c & 15, rl = c >> 4;
    const int e = e0 + 4 * q;
    float4 bs = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 va[kWrRows], vb[kWrRows];
    auto load = [&](float4 (&v)[kWrRows], int i) {
      const int tk = (kb0 + i) * 64;
#pragma unroll
      for (int m = 0; m < kWrRows; ++m)
        v[m] = load4(g.dl, tk + rl + 16 * m, g.T, e < e0 + Ec ? e : g.E, g.E);
    };
    int stage = 0;
    uint32_t phase = 0;
    auto put = [&](const float4 (&v)[kWrRows]) -> bool {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) return false;
      uint8_t* bh = ring + stage * kWrStage + 2 * kChunk;
#pragma unroll
      for (int m = 0; m < kWrRows; ++m) {
        bs.x += v[m].x;
        bs.y += v[m].y;
        bs.z += v[m].z;
        bs.w += v[m].w;
        uint2 hi, lo;
        split4(v[m], hi, lo);
        const int off = sw128(rl + 16 * m, q >> 1, q & 1);
        *reinterpret_cast<uint2*>(bh + off) = hi;
        *reinterpret_cast<uint2*>(bh + kChunk + off) = lo;
      }
      fence_proxy_async_smem();  // the generic stores before the tensor cores' reads
      mbar_arrive(saddr(&full[stage]));
      if (++stage == kWrStages) {
        stage = 0;
        phase ^= 1u;
      }
      return true;
    };
    // two blocks in flight: the next block's loads are issued before this one is stored
    bool ok = true;
    if (nkb > 0) load(va, 0);
    for (int i = 0; i < nkb && ok; i += 2) {
      if (i + 1 < nkb) load(vb, i + 1);
      ok = put(va);
      if (ok && i + 1 < nkb) {
        if (i + 2 < nkb) load(va, i + 2);
        ok = put(vb);
      }
    }
    // the CTA's d_bias partial: per expert, the 16 row lanes' sums in row-lane order
    *reinterpret_cast<float4*>(bias_part + 4 * c) = bs;
    asm volatile("bar.sync 1, %0;" ::"n"(kWrConv) : "memory");
    if (c < 64) {
      float v = 0.f;
      for (int r = 0; r < 16; ++r) v += bias_part[4 * (16 * r + (c >> 2)) + (c & 3)];
      cta_bias[c] = v;
    }
    // ---- the partial tile to shared memory (warps 2-5): part[row j][expert e - e0]
    if (warp < 6) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(accf), 0, abort_flag, g.status, g.limit_ns);
      w = __shfl_sync(0xffffffffu, w, 0);
      tc_fence_after();
      const bool have = w && nkb > 0 && *abort_flag == 0;
      const int qw = warp & 3;
      float* prow = (float*)ring + (32 * qw + lane) * kWrPs;
      for (int c0 = 0; c0 < NE; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * qw) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          *reinterpret_cast<float4*>(prow + c0 + k) =
              have ? make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                                 __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // every rank's partial tile and bias sums are in its shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kWrTmemCols);
  }
  if (*abort_flag == 0) {
    const int per = 128 / S, rb = (int)rank * per;
    const float* part = (const float*)ring;
    for (int i = tid; i < per * Ec; i += kWrThreads) {
      const int r = rb + i / Ec, e = i % Ec;
      const uint32_t la = saddr(part + r * kWrPs + e);
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += ld_dsmem_f32(map_rank(la, (uint32_t)q));  // rank order
      const int j = j0 + r;
      if (j < g.d) g.d_w_r[(size_t)j * g.E + e0 + e] = v;
    }
    if (g.d_bias != nullptr && mtile == 0 && rank == 0) {
      for (int e = tid; e < Ec; e += kWrThreads) {
        const uint32_t la = saddr(cta_bias + e);
        float v = 0.f;
        for (int q = 0; q < S; ++q) v += ld_dsmem_f32(map_rank(la, (uint32_t)q));
        g.d_bias[e0 + e] = v;
      }
    }
  }
  cluster_sync();  // the peers' tiles have been read; they may exit
}

// ------------------------------------------------------------------ d_x
constexpr int kDxThreads = 256;
constexpr int kDxAtomA = 128 * 128;  // 16 KB: 128 token rows x 64 experts
constexpr int kDxAtomB = 128 * 128;  // 16 KB: 128 columns of d x 64 experts
constexpr int kDxTmemCols = 128;
constexpr int kDxPs = 64 + 4;  // row stride (floats) of a staged 64-column half
constexpr uint32_t kDxIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);  // A and B K-major, M = N = 128
static_assert(128 * kDxPs * 4 <= 2 * kDxAtomA + kDxAtomB, "a staged half fits the operands");

struct DxArgs {
  const float* dl;
  bf16* d_x;
  int T, d, E;
  int natoms;  // 64-expert atoms: ceil(E / 64)
  int ksteps;  // 16-expert MMA steps: ceil(E / 16)
  unsigned* status;
  unsigned long long limit_ns;
};

__global__ void __launch_bounds__(kDxThreads) router_dx_tc_kernel(
    const __grid_constant__ CUtensorMap tmW, const DxArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const int NA = g.natoms;
  uint8_t* a_hi = align1024(smem_raw);
  uint8_t* a_lo = a_hi + NA * kDxAtomA;
  uint8_t* bsm = a_lo + NA * kDxAtomA;
  uint64_t* bar_b = (uint64_t*)(bsm + NA * kDxAtomB);
  uint64_t* bar_acc = bar_b + 1;
  uint32_t* tmem_slot = (uint32_t*)(bar_b + 2);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * 128, j0 = blockIdx.y * 128;

  if (tid == 32) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmW) : "memory");
  if (tid == 0) {
    mbar_init(saddr(bar_b), 1);
    mbar_init(saddr(bar_acc), 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc<1>(saddr(tmem_slot), kDxTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the previous kernel in the stream has completed (dL/dl and d_x written)
  pdl_trigger();
  if (tid == 0) {
    mbar_expect_tx(saddr(bar_b), (uint32_t)(NA * kDxAtomB));
    for (int c = 0; c < NA; ++c)
      tma_load_2d(saddr(bsm + c * kDxAtomB), &tmW, c * 64, j0, saddr(bar_b));
  }
  // the tile's d_x values, loaded now so that their latency passes under the conversion and
  // the MMAs: thread tid owns columns j0 + 64 h + 8 (tid % 8) .. + 7 of rows tid / 8 + 32 m
  const int cu = tid & 7, rr = tid >> 3;
  uint4 old[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int t = t0 + rr + 32 * m, j = j0 + 64 * h + 8 * cu;
      old[h][m] = (t < g.T && j < g.d)
                      ? *reinterpret_cast<const uint4*>(g.d_x + (size_t)t * g.d + j)
                      : make_uint4(0, 0, 0, 0);
    }
  // A: the tile's dL/dl rows as hi / lo terms, K-major, 128-byte swizzle; one float4 per
  // thread and unit, 8 units in flight
  const int nq = NA * 16, units = 128 * nq;
  for (int u0 = tid; u0 < units; u0 += 8 * kDxThreads) {
    float4 v[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kDxThreads, r = u / nq, q = u - r * nq;
      v[m] = load4(g.dl, u < units ? t0 + r : g.T, g.T, 4 * q, g.E);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kDxThreads, r = u / nq, q = u - r * nq;
      if (u < units) {
        uint2 hi, lo;
        split4(v[m], hi, lo);
        const int off = (q >> 4) * kDxAtomA + sw128(r, (q >> 1) & 7, q & 1);
        *reinterpret_cast<uint2*>(a_hi + off) = hi;
        *reinterpret_cast<uint2*>(a_lo + off) = lo;
      }
    }
  }
  fence_proxy_async_smem();  // the generic stores before the tensor cores' reads
  __syncthreads();
  if (tid == 0) {
    if (mbar_wait(saddr(bar_b), 0, abort_flag, g.status, g.limit_ns)) {
      tc_fence_after();
      for (int k = 0; k < g.ksteps; ++k) {
        const uint32_t oa = (uint32_t)((k >> 2) * kDxAtomA + (k & 3) * 32);
        const uint32_t ob = (uint32_t)((k >> 2) * kDxAtomB + (k & 3) * 32);
        const uint64_t bd = desc_sw128(saddr(bsm) + ob, 16, 1024);
        tc_mma<1>(tmem, desc_sw128(saddr(a_hi) + oa, 16, 1024), bd, kDxIdesc, k > 0 ? 1u : 0u);
        tc_mma<1>(tmem, desc_sw128(saddr(a_lo) + oa, 16, 1024), bd, kDxIdesc, 1u);
      }
    }
    tc_commit<1>(saddr(bar_acc));  // arrives at once if nothing was issued
  }
  __syncwarp();
  int w = 0;
  if (lane == 0) w = mbar_wait(saddr(bar_acc), 0, abort_flag, g.status, g.limit_ns);
  w = __shfl_sync(0xffffffffu, w, 0);
  tc_fence_after();
  const bool ok = w && *abort_flag == 0;
  // epilogue, per 64-column half: warp w copies TMEM lanes 32 (w % 4) ... (its 32 token
  // rows), columns 64 h + 32 (w / 4) ... + 31, into the staging rows (the operands' shared
  // memory, free once the MMAs completed); then each thread adds its staged sums to the d_x
  // values it loaded and stores them: d_x[t, j] = bf16(d_x[t, j] + sum)
  float* stg = (float*)a_hi;
  const int qw = warp & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    {
      uint32_t v[32];
      const int cs = 64 * h + 32 * (warp >> 2);
      tmem_ld32(tmem + ((uint32_t)(32 * qw) << 16) + (uint32_t)cs, v);
      tmem_ld_wait();
      float* dst = stg + (32 * qw + lane) * kDxPs + 32 * (warp >> 2);
#pragma unroll
      for (int k = 0; k < 32; k += 4)
        *reinterpret_cast<float4*>(dst + k) =
            make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]),
                        __uint_as_float(v[k + 2]), __uint_as_float(v[k + 3]));
    }
    __syncthreads();
    if (ok) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int row = rr + 32 * m, t = t0 + row, j = j0 + 64 * h + 8 * cu;
        if (t < g.T && j < g.d) {
          const float* src = stg + row * kDxPs + 8 * cu;
          const float4 a = *reinterpret_cast<const float4*>(src);
          const float4 b = *reinterpret_cast<const float4*>(src + 4);
          float f[8];
          unpack16(old[h][m], f, bf16());
          f[0] += a.x, f[1] += a.y, f[2] += a.z, f[3] += a.w;
          f[4] += b.x, f[5] += b.y, f[6] += b.z, f[7] += b.w;
          *reinterpret_cast<uint4*>(g.d_x + (size_t)t * g.d + j) = pack16(f, bf16());
        }
      }
    }
    __syncthreads();  // the half has been read before the next one is staged
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kDxTmemCols);
  }
}

// ------------------------------------------------------------------ d_x, streamed (E <= 128)
// One CTA per 128-token tile (and, when there are fewer tiles than SMs, per group of column
// tiles): the tile's dL/dl rows are converted once, then the CTA streams its column tiles.
// Warp 0 loads the d_x tiles by TMA into a 3-stage ring (128-byte swizzle, two 64-column
// halves); warp 1 loads the W_r tile by TMA and issues the MMAs into one of two 128-column
// accumulators; warps 2-5 add each accumulator row to its d_x row in shared memory (the
// swizzle puts 8 consecutive rows' units in different banks), and one thread stores the tile
// back by TMA. A d_x stage is reloaded once the store that read it has finished reading.
constexpr int kPxThreads = 192;
constexpr int kPxDxStages = 3;
constexpr int kPxTile = 128 * 128 * 2;  // 32 KB: a 128 x 128 bf16 tile, two 64-column halves
constexpr int kPxTmemCols = 256;        // two 128-column accumulators

struct PxArgs {
  const float* dl;
  int T, d, E;
  int natoms, ksteps;
  int ntiles;  // column tiles of 128: ceil(d / 128)
  int per;     // column tiles per CTA (blockIdx.y takes tiles [per y, per (y + 1)))
  unsigned* status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1,
                                             uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   (uint64_t)map),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {  // all but N groups have read their source
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {  // all but N groups have completed
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kPxThreads, 1) router_dx_tc_stream_kernel(
    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmD,
    const PxArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const int NA = g.natoms;
  uint8_t* a_hi = align1024(smem_raw);
  uint8_t* a_lo = a_hi + NA * kDxAtomA;
  uint8_t* bsm = a_lo + NA * kDxAtomA;  // one W_r tile: NA atoms of 16 KB
  uint8_t* dxs = bsm + NA * kDxAtomB;   // the d_x ring
  uint64_t* bars = (uint64_t*)(dxs + kPxDxStages * kPxTile);
  uint64_t* b_full = bars;         // the W_r tile landed
  uint64_t* b_empty = bars + 1;    // the MMAs reading it completed
  uint64_t* acc_full = bars + 2;   // [2] accumulator complete
  uint64_t* acc_empty = bars + 4;  // [2] the 4 epilogue warps have read it
  uint64_t* dx_full = bars + 6;    // [3] d_x tile landed
  uint64_t* dx_empty = bars + 9;   // [3] the store of the tile in it has read it
  uint32_t* tmem_slot = (uint32_t*)(bars + 12);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * 128;
  const int jt0 = blockIdx.y * g.per;
  const int nt = min(g.ntiles, jt0 + g.per) - jt0;  // >= 1 (the host sizes the grid so)

  if (tid == 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmW) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmD) : "memory");
  }
  if (tid == 0) {
    mbar_init(saddr(b_full), 1);
    mbar_init(saddr(b_empty), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&acc_full[b]), 1);
      mbar_init(saddr(&acc_empty[b]), 4);
    }
    for (int s = 0; s < kPxDxStages; ++s) {
      mbar_init(saddr(&dx_full[s]), 1);
      mbar_init(saddr(&dx_empty[s]), 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) tmem_alloc<1>(saddr(tmem_slot), kPxTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the previous kernel in the stream has completed (dL/dl and d_x written)
  pdl_trigger();
  auto load_dx = [&](int n) {  // tile n of this CTA into stage n % 3
    const int sd = n % kPxDxStages, j = (jt0 + n) * 128;
    const uint32_t fb = saddr(&dx_full[sd]), dst = saddr(dxs + sd * kPxTile);
    mbar_expect_tx(fb, kPxTile);
    tma_load_2d(dst, &tmD, j, t0, fb);
    tma_load_2d(dst + kPxTile / 2, &tmD, j + 64, t0, fb);
  };
  auto load_w = [&](int n) {
    const uint32_t fb = saddr(b_full);
    mbar_expect_tx(fb, (uint32_t)(NA * kDxAtomB));
    for (int c = 0; c < NA; ++c)
      tma_load_2d(saddr(bsm + c * kDxAtomB), &tmW, c * 64, (jt0 + n) * 128, fb);
  };
  if (tid == 0) {  // the first d_x tiles and W_r tile are on their way during the conversion
    for (int n = 0; n < nt && n < kPxDxStages; ++n) load_dx(n);
    load_w(0);
  }
  // A: the tile's dL/dl rows as hi / lo terms, K-major, 128-byte swizzle
  const int nq = NA * 16, units = 128 * nq;
  for (int u0 = tid; u0 < units; u0 += 8 * kPxThreads) {
    float4 v[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kPxThreads, r = u / nq, q = u - r * nq;
      v[m] = load4(g.dl, u < units ? t0 + r : g.T, g.T, 4 * q, g.E);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kPxThreads, r = u / nq, q = u - r * nq;
      if (u < units) {
        uint2 hi, lo;
        split4(v[m], hi, lo);
        const int off = (q >> 4) * kDxAtomA + sw128(r, (q >> 1) & 7, q & 1);
        *reinterpret_cast<uint2*>(a_hi + off) = hi;
        *reinterpret_cast<uint2*>(a_lo + off) = lo;
      }
    }
  }
  fence_proxy_async_smem();  // the generic stores before the tensor cores' reads
  __syncthreads();

  if (warp == 0) {
    // ---- d_x loads of tiles 3, 4, ...: stage n % 3 once the store of tile n - 3 read it
    for (int n = kPxDxStages; n < nt; ++n) {
      int w = 0;
      if (lane == 0)
        w = mbar_wait(saddr(&dx_empty[n % kPxDxStages]), ((n / kPxDxStages) & 1) ^ 1u,
                      abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (lane == 0) load_dx(n);
      __syncwarp();
    }
  } else if (warp == 1) {
    // ---- MMAs of tile n into accumulator n % 2, then the W_r tile of tile n + 1
    for (int n = 0; n < nt; ++n) {
      const int buf = n & 1;
      int w = 0;
      if (lane == 0)
        w = mbar_wait(saddr(b_full), (uint32_t)(n & 1), abort_flag, g.status, g.limit_ns) &&
            mbar_wait(saddr(&acc_empty[buf]), (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag,
                      g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t d_acc = tmem + (uint32_t)(128 * buf);
        for (int k = 0; k < g.ksteps; ++k) {
          const uint32_t oa = (uint32_t)((k >> 2) * kDxAtomA + (k & 3) * 32);
          const uint32_t ob = (uint32_t)((k >> 2) * kDxAtomB + (k & 3) * 32);
          const uint64_t bd = desc_sw128(saddr(bsm) + ob, 16, 1024);
          tc_mma<1>(d_acc, desc_sw128(saddr(a_hi) + oa, 16, 1024), bd, kDxIdesc,
                    k > 0 ? 1u : 0u);
          tc_mma<1>(d_acc, desc_sw128(saddr(a_lo) + oa, 16, 1024), bd, kDxIdesc, 1u);
        }
        tc_commit<1>(saddr(&acc_full[buf]));
        tc_commit<1>(saddr(b_empty));
      }
      __syncwarp();
      if (n + 1 < nt) {
        if (lane == 0)
          w = mbar_wait(saddr(b_empty), (uint32_t)(n & 1), abort_flag, g.status, g.limit_ns);
        if (!__shfl_sync(0xffffffffu, w, 0)) break;
        if (lane == 0) load_w(n + 1);
        __syncwarp();
      }
    }
  } else {
    // ---- epilogue (warps 2-5): warp w owns TMEM lanes 32 (w % 4) ..., the tile's token rows
    // r = 32 (w % 4) + lane; d_x[t, j] = bf16(d_x[t, j] + sum) in place, then the TMA store.
    // Every warp takes every tile (no early exit: the named barrier needs all four).
    const int qw = warp & 3, r = 32 * qw + lane;
    for (int n = 0; n < nt; ++n) {
      const int buf = n & 1, sd = n % kPxDxStages;
      int w = 0;
      if (lane == 0)
        w = mbar_wait(saddr(&acc_full[buf]), (uint32_t)((n >> 1) & 1), abort_flag, g.status,
                      g.limit_ns) &&
            mbar_wait(saddr(&dx_full[sd]), (uint32_t)((n / kPxDxStages) & 1), abort_flag,
                      g.status, g.limit_ns);
      w = __shfl_sync(0xffffffffu, w, 0);
      tc_fence_after();
      uint8_t* tile = dxs + sd * kPxTile;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * qw) << 16) + (uint32_t)(128 * buf + c0), v);
        tmem_ld_wait();
        if (w) {
          uint8_t* half = tile + (c0 >> 6) * (kPxTile / 2);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4* p = reinterpret_cast<uint4*>(half + sw128(r, ((c0 & 63) >> 3) + k, 0));
            float f[8];
            unpack16(*p, f, bf16());
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] += __uint_as_float(v[8 * k + i]);
            *p = pack16(f, bf16());
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(saddr(&acc_empty[buf]));
      fence_proxy_async_smem();  // the generic stores before the TMA store reads them
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0) {
        if (*abort_flag == 0) {
          const int j = (jt0 + n) * 128;
          tma_store_2d(&tmD, j, t0, saddr(tile));
          if (j + 64 < g.d) tma_store_2d(&tmD, j + 64, t0, saddr(tile + kPxTile / 2));
        }
        bulk_commit();
        bulk_wait_read<1>();  // the store of tile n - 1 has read its stage
        if (n >= 1) mbar_arrive(saddr(&dx_empty[(n - 1) % kPxDxStages]));
      }
      __syncwarp();
    }
    if (warp == 2 && lane == 0) bulk_wait<0>();  // every store has completed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kPxTmemCols);
  }
}

bool aligned16p(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Clusters of S CTAs of the d_W_r kernel that can be resident at once: clusters stay inside
// one GPC, so this can be below 2 SMs / S. Cached per device and S; the kernel's
// shared-memory attribute is set first.
int resident_clusters(int S) {
  struct Entry {
    int dev, S, n;
  };
  static std::mutex mu;
  static Entry cache[32];
  static int used = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].S == S) return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S);
  cfg.blockDim = dim3(kWrThreads);
  cfg.dynamicSmemBytes = (size_t)kWrSmem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = (unsigned)S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)router_dwr_tc_kernel, &cfg) !=
          cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (used < 32) cache[used++] = Entry{dev, S, n};
  return n;
}

}  // namespace

// The tensor-core forms take routers of 17..256 experts with E % 8 == 0 and 16-byte-aligned
// operands (d % 64 == 0 holds for every shape); *used = false leaves the call to the
// CUDA-core forms.
moe_status launch_router_dwr_tc(const moe_shape& s, const void* x, const float* d_logits,
                                float* d_w_r, float* d_bias, cudaStream_t st, bool* used) {
  *used = false;
  const int T = s.T, d = s.d, E = s.E;
  if (E <= 16 || E > 256 || E % 8 != 0 || T < 1) return MOE_OK;
  if (!aligned16p(x) || !aligned16p(d_logits)) return MOE_OK;
  CUtensorMap mx;
  {
    const uint64_t dims[2] = {(uint64_t)d, (uint64_t)T}, str[1] = {(uint64_t)d * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_map(&mx, x, 2, dims, str, box)) return MOE_OK;
  }
  DwrArgs a;
  a.dl = d_logits;
  a.d_w_r = d_w_r;
  a.d_bias = d_bias;
  a.T = T;
  a.d = d;
  a.E = E;
  a.nchunks = (E + 63) / 64;
  a.kb_total = (T + 63) / 64;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  if (cudaFuncSetAttribute(router_dwr_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kWrSmem) != cudaSuccess)
    return MOE_ERR_CUDA;
  // clusters of S CTAs splitting the tokens: S from 8, 4, 2, 1, the one with the fewest
  // rounds of resident clusters per unit of work, ceil(clusters / resident(S)) / S (ties to
  // the fewer rounds)
  const int clusters = ((d + 127) / 128) * a.nchunks;
  int best_S = 1;
  long long best_rounds = 0;
  for (int S = 8; S >= 1; S >>= 1) {
    const int n = resident_clusters(S);
    const long long rounds = (clusters + n - 1) / n;
    if (S == 8 || rounds * best_S < best_rounds * S ||
        (rounds * best_S == best_rounds * S && rounds < best_rounds)) {
      best_S = S;
      best_rounds = rounds;
    }
  }
  a.S = best_S;
  launch_begin(K_ROUTER_DWR, st);
  if (launch_kernel(router_dwr_tc_kernel, dim3((unsigned)(clusters * best_S)), dim3(kWrThreads),
                    (size_t)kWrSmem, st, (unsigned)best_S, mx, a) != cudaSuccess)
    return MOE_ERR_CUDA;
  *used = true;
  return launch_end(K_ROUTER_DWR, st);
}

moe_status launch_router_dx_tc(const moe_shape& s, const void* w_r, const float* d_logits,
                               void* d_x, cudaStream_t st, bool* used) {
  *used = false;
  const int T = s.T, d = s.d, E = s.E;
  if (E <= 16 || E > 256 || E % 8 != 0 || T < 1) return MOE_OK;
  if (!aligned16p(w_r) || !aligned16p(d_logits) || !aligned16p(d_x)) return MOE_OK;
  CUtensorMap mw;
  {
    const uint64_t dims[2] = {(uint64_t)E, (uint64_t)d}, str[1] = {(uint64_t)E * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_map(&mw, w_r, 2, dims, str, box)) return MOE_OK;
  }
  if (E <= 128) {  // the streamed form: one conversion per token tile
    CUtensorMap md;
    const uint64_t dims[2] = {(uint64_t)d, (uint64_t)T}, str[1] = {(uint64_t)d * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_map(&md, d_x, 2, dims, str, box)) return MOE_OK;
    PxArgs p;
    p.dl = d_logits;
    p.T = T;
    p.d = d;
    p.E = E;
    p.natoms = (E + 63) / 64;
    p.ksteps = (E + 15) / 16;
    p.ntiles = (d + 127) / 128;
    p.status = device_status_ptr();
    p.limit_ns = kWaitLimitNs;
    const int rows = (T + 127) / 128;
    int groups = rows >= sm_count() ? 1 : sm_count() / rows;  // column groups per token tile
    if (groups > p.ntiles) groups = p.ntiles;
    p.per = (p.ntiles + groups - 1) / groups;
    groups = (p.ntiles + p.per - 1) / p.per;  // every group has a tile
    const size_t smem = (size_t)(1024 + p.natoms * (2 * kDxAtomA + kDxAtomB) +
                                 kPxDxStages * kPxTile + 128);
    if (cudaFuncSetAttribute(router_dx_tc_stream_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_begin(K_ROUTER_DX, st);
    if (launch_kernel(router_dx_tc_stream_kernel, dim3((unsigned)rows, (unsigned)groups),
                      dim3(kPxThreads), smem, st, 1, mw, md, p) != cudaSuccess)
      return MOE_ERR_CUDA;
    *used = true;
    return launch_end(K_ROUTER_DX, st);
  }
  DxArgs a;
  a.dl = d_logits;
  a.d_x = (bf16*)d_x;
  a.T = T;
  a.d = d;
  a.E = E;
  a.natoms = (E + 63) / 64;
  a.ksteps = (E + 15) / 16;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  const size_t smem = (size_t)(1024 + a.natoms * (2 * kDxAtomA + kDxAtomB) + 32);
  if (cudaFuncSetAttribute(router_dx_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const dim3 grid((unsigned)((T + 127) / 128), (unsigned)((d + 127) / 128));
  launch_begin(K_ROUTER_DX, st);
  if (launch_kernel(router_dx_tc_kernel, grid, dim3(kDxThreads), smem, st, 1, mw, a) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  *used = true;
  return launch_end(K_ROUTER_DX, st);
}

}  // namespace moe
