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
// d_W_r (router_dwr_tc_kernel): D[j, e] = sum_t x[t, j] dL/dl[t, e], 128 columns of x on the
// MMA's M and the experts on N (E rounded up to 32); K = tokens in blocks of 64. A = x[t, j]
// tiles by TMA, MN-major (two [64 t][64 j] 128-byte-swizzled chunks); B = dL/dl rows
// converted to the hi / lo terms by eight converter warps and written in the layout TMA
// would give a [64 t][64 e] box (MN-major, 128-byte swizzle). The tokens are split over the
// S CTAs of a cluster (contiguous ranges of whole blocks); after the last MMA each CTA
// copies its partial tile to shared memory and, after a cluster barrier, CTA q adds the S
// partials of rows [q 128/S, (q+1) 128/S) in rank order through distributed shared memory
// (the same fp32 sums in the same order on every run). The converters also add up their
// fp32 values per expert in token order; d_bias is the cluster's rank-ordered sum of those.
// Roles (320 threads): warp 0 issues the x loads, warp 1 the MMAs, warps 2-9 convert; warps
// 2-5 read the accumulator (warp w may read TMEM lanes 32 (w % 4) ...).
//
// d_x (router_dx_tc_kernel): D[t, j] = sum_e dL/dl[t, e] W_r[j, e], 128 tokens on M and 128
// columns of d on N, K = experts (at most 256, so one shot: no ring). A = the tile's dL/dl
// rows as hi and lo terms (K-major, converted by all threads), B = W_r rows by TMA (K-major:
// W_r is [d, E] with E innermost). The epilogue adds the fp32 sums to the bf16 d_x rows and
// rounds once, as the CUDA-core form does.
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

// 16-byte unit u (of 8) of row r inside a 128-byte-swizzled span of 8-row groups: the unit
// index is XORed with the row's index inside its group of 8.
__device__ __forceinline__ int sw128(int r, int u) { return r * 128 + ((u ^ (r & 7)) << 4); }

// Eight fp32 values as two bf16 vectors hi and lo with v = hi + lo + (|error| <= 2^-16 |v|).
__device__ __forceinline__ void split8(const float (&v)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    const float b0 = __uint_as_float(h[i] << 16), b1 = __uint_as_float(h[i] & 0xffff0000u);
    l[i] = pack_bf16x2(v[2 * i] - b0, v[2 * i + 1] - b1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Eight consecutive dL/dl values of token t from expert e (E % 8 == 0: all in or all out).
__device__ __forceinline__ void load8(const float* __restrict__ dl, int t, int T, int e, int E,
                                      float (&v)[8]) {
  if (t < T && e < E) {
    const float4* p = reinterpret_cast<const float4*>(dl + (size_t)t * E + e);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z,
    v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return (uint8_t*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// ------------------------------------------------------------------ d_W_r and d_bias
constexpr int kWrThreads = 320;
constexpr int kWrConv = 256;  // converter threads (warps 2-9)
constexpr int kWrMaxStages = 6;
constexpr int kWrTmemCols = 256;

struct DwrArgs {
  const float* dl;
  float* d_w_r;
  float* d_bias;
  int T, d, E;
  int NE;           // the MMA's N: E rounded up to 32
  int nbc;          // 64-expert chunks of B: ceil(E / 64)
  int S;            // CTAs of a cluster splitting the tokens
  int kb_total;     // blocks of 64 tokens: ceil(T / 64)
  int stages, stage_bytes;
  int ps;           // row stride (floats) of the partial tile in shared memory
  unsigned* status;
  unsigned long long limit_ns;
};

// NQ = 8 nbc units of 8 experts per token row; a converter thread owns unit q = c % NQ of the
// rows rl, rl + R, ... (rl = c / NQ < R = 256 / NQ) of every block: ROWS rows at most.
template <int NQ>
__global__ void __launch_bounds__(kWrThreads, 1)
    router_dwr_tc_kernel(const __grid_constant__ CUtensorMap tmX, const DwrArgs g) {
  constexpr int R = kWrConv / NQ;
  constexpr int ROWS = (64 + R - 1) / R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = align1024(smem_raw);
  float* bias_part = (float*)(ring + g.stages * g.stage_bytes);  // [256 converters][8]
  float* cta_bias = bias_part + kWrConv * 8;                      // [256]
  uint64_t* full = (uint64_t*)(cta_bias + 256);
  uint64_t* empty = full + kWrMaxStages;
  uint64_t* accf = empty + kWrMaxStages;
  uint32_t* tmem_slot = (uint32_t*)(accf + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = g.S, ST = g.stages, SB = g.stage_bytes;
  const uint32_t rank = cluster_rank();  // 0 without a cluster
  const int mtile = (int)cluster_id_x();
  const int j0 = mtile * 128;
  const int kb0 = (int)((long long)rank * g.kb_total / S);
  const int nkb = (int)((long long)(rank + 1) * g.kb_total / S) - kb0;

  if (tid == 32) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmX) : "memory");
  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
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
        const uint32_t a = saddr(ring + stage * SB);
        const int tk = (kb0 + i) * 64;
        mbar_expect_tx(fb, 2 * kChunk);
        tma_load_2d(a, &tmX, j0, tk, fb);
        tma_load_2d(a + kChunk, &tmX, j0 + 64, tk, fb);
      }
      __syncwarp();
      if (++stage == ST) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issue: per block, 4 steps of 16 tokens, each as hi then lo
    // A (MN-major): 64-column chunks 8 KB apart, 8-row groups 1 KB apart, a step = 16 rows.
    // B (MN-major): 64-expert chunks 8 KB apart, the same row geometry.
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           ((uint32_t)(g.NE >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&full[stage]), phase, abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a = saddr(ring + stage * SB);
        const uint32_t bh = a + 2 * kChunk, bl = bh + (uint32_t)(g.nbc * kChunk);
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
      if (++stage == ST) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0) tc_commit<1>(saddr(accf));  // arrives at once if nothing was issued
    __syncwarp();
  } else {
    // ---- converters: dL/dl rows -> hi / lo bf16 in the B slots; fp32 column sums for d_bias
    const int c = tid - 64;
    const int q = c % NQ, rl = c / NQ;
    const bool active = rl < R;
    const int e = 8 * q;
    float bs[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) bs[k] = 0.f;
    float va[ROWS][8], vb[ROWS][8];
    auto load = [&](float (&v)[ROWS][8], int i) {
      const int tk = (kb0 + i) * 64;
#pragma unroll
      for (int m = 0; m < ROWS; ++m) {
        const int r = rl + m * R;
        load8(g.dl, (active && r < 64) ? tk + r : g.T, g.T, e, g.E, v[m]);
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto put = [&](float (&v)[ROWS][8]) -> bool {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) return false;
      if (active) {
        uint8_t* bh = ring + stage * SB + 2 * kChunk;
        uint8_t* bl = bh + g.nbc * kChunk;
#pragma unroll
        for (int m = 0; m < ROWS; ++m) {
          const int r = rl + m * R;
          if (r < 64) {
#pragma unroll
            for (int k = 0; k < 8; ++k) bs[k] += v[m][k];
            uint4 hi, lo;
            split8(v[m], hi, lo);
            const int off = (q >> 3) * kChunk + sw128(r, q & 7);
            *reinterpret_cast<uint4*>(bh + off) = hi;
            *reinterpret_cast<uint4*>(bl + off) = lo;
          }
        }
        fence_proxy_async_smem();  // the generic stores before the tensor cores' reads
      }
      mbar_arrive(saddr(&full[stage]));
      if (++stage == ST) {
        stage = 0;
        phase ^= 1u;
      }
      return true;
    };
    // two blocks in flight: the next block's loads are issued before this one is stored
    if (nkb > 0) load(va, 0);
    for (int i = 0; i < nkb && ok; i += 2) {
      if (i + 1 < nkb) load(vb, i + 1);
      ok = put(va);
      if (ok && i + 1 < nkb) {
        if (i + 2 < nkb) load(va, i + 2);
        ok = put(vb);
      }
    }
    // the CTA's d_bias partial: per expert, the converters' sums in converter order
    if (active) {
#pragma unroll
      for (int k = 0; k < 8; ++k) bias_part[c * 8 + k] = bs[k];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kWrConv) : "memory");
    for (int x = c; x < g.E; x += kWrConv) {
      float v = 0.f;
      for (int r = 0; r < R; ++r) v += bias_part[(r * NQ + (x >> 3)) * 8 + (x & 7)];
      cta_bias[x] = v;
    }
    // ---- the partial tile to shared memory (warps 2-5): part[row j][expert e]
    if (warp < 6) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(accf), 0, abort_flag, g.status, g.limit_ns);
      w = __shfl_sync(0xffffffffu, w, 0);
      tc_fence_after();
      const bool have = w && nkb > 0 && *abort_flag == 0;
      const int qw = warp & 3;
      float* prow = (float*)ring + (32 * qw + lane) * g.ps;
      for (int c0 = 0; c0 < g.NE; c0 += 32) {
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
    for (int i = tid; i < per * g.E; i += kWrThreads) {
      const int r = rb + i / g.E, e = i % g.E;
      const uint32_t la = saddr(part + r * g.ps + e);
      float v = 0.f;
      for (int q = 0; q < S; ++q) v += ld_dsmem_f32(map_rank(la, (uint32_t)q));  // rank order
      const int j = j0 + r;
      if (j < g.d) g.d_w_r[(size_t)j * g.E + e] = v;
    }
    if (g.d_bias != nullptr && mtile == 0 && rank == 0) {
      for (int e = tid; e < g.E; e += kWrThreads) {
        const uint32_t la = saddr(cta_bias + e);
        float v = 0.f;
        for (int q = 0; q < S; ++q) v += ld_dsmem_f32(map_rank(la, (uint32_t)q));
        g.d_bias[e] = v;
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
constexpr uint32_t kDxIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);  // A and B K-major, M = N = 128

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
  // the epilogue's d_x values (warp w: its 32 token rows, columns 64 (w / 4) ... + 63), loaded
  // now so that their latency passes under the conversion and the MMAs
  const int qw = warp & 3, r = 32 * qw + lane, t = t0 + r, cb = j0 + 64 * (warp >> 2);
  uint4 old[8];
#pragma unroll
  for (int s = 0; s < 8; ++s)
    old[s] = (t < g.T && cb + 8 * s < g.d)
                 ? *reinterpret_cast<const uint4*>(g.d_x + (size_t)t * g.d + cb + 8 * s)
                 : make_uint4(0, 0, 0, 0);
  // A: the tile's dL/dl rows as hi / lo terms, K-major, 128-byte swizzle; 8 units in flight
  const int nq = NA * 8, units = 128 * nq;
  for (int u0 = tid; u0 < units; u0 += 8 * kDxThreads) {
    float v[8][8];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kDxThreads, r = u / nq, q = u - r * nq;
      load8(g.dl, u < units ? t0 + r : g.T, g.T, 8 * q, g.E, v[m]);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int u = u0 + m * kDxThreads, r = u / nq, q = u - r * nq;
      if (u < units) {
        uint4 hi, lo;
        split8(v[m], hi, lo);
        const int off = (q >> 3) * kDxAtomA + sw128(r, q & 7);
        *reinterpret_cast<uint4*>(a_hi + off) = hi;
        *reinterpret_cast<uint4*>(a_lo + off) = lo;
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
  // epilogue: warp w reads TMEM lanes 32 (w % 4) ... (its 32 token rows), columns
  // 64 (w / 4) ... + 63; d_x[t, j] = bf16(d_x[t, j] + sum)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(32 * qw) << 16) + (uint32_t)(64 * (warp >> 2) + 32 * h), v);
    tmem_ld_wait();
    if (ok && t < g.T) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int j = cb + 32 * h + 8 * s;
        if (j < g.d) {
          float f[8];
          unpack16(old[4 * h + s], f, bf16());
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] += __uint_as_float(v[8 * s + k]);
          *reinterpret_cast<uint4*>(g.d_x + (size_t)t * g.d + j) = pack16(f, bf16());
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kDxTmemCols);
  }
}

bool aligned16p(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Clusters of S CTAs of `kern` (kWrThreads threads, `smem` bytes) that can be resident at
// once: clusters stay inside one GPC, so this can be below SMs / S. Cached per device,
// kernel, S and shared-memory size; the kernel's shared-memory attribute is set first.
int resident_clusters(const void* kern, int smem, int S) {
  struct Entry {
    const void* kern;
    int dev, S, smem, n;
  };
  static std::mutex mu;
  static Entry cache[32];
  static int used = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].kern == kern && cache[i].dev == dev && cache[i].S == S && cache[i].smem == smem)
      return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S);
  cfg.blockDim = dim3(kWrThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = (unsigned)S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (used < 32) cache[used++] = Entry{kern, dev, S, smem, n};
  return n;
}

// Launches the d_W_r kernel over `tiles` column tiles with clusters of S CTAs splitting the
// tokens: S from 8, 4, 2, 1, the one with the fewest rounds of resident clusters per unit of
// work, ceil(tiles / resident(S)) / S (ties to the fewer rounds).
template <int NQ>
cudaError_t launch_dwr(int tiles, size_t smem, cudaStream_t st, const CUtensorMap& m,
                       DwrArgs a) {
  auto kern = router_dwr_tc_kernel<NQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int best_S = 1;
  long long best_rounds = 0;
  for (int S = 8; S >= 1; S >>= 1) {
    const int n = resident_clusters((const void*)kern, (int)smem, S);
    const long long rounds = (tiles + n - 1) / n;
    // rounds / S < best_rounds / best_S, or equal with fewer rounds
    if (S == 8 || rounds * best_S < best_rounds * S ||
        (rounds * best_S == best_rounds * S && rounds < best_rounds)) {
      best_S = S;
      best_rounds = rounds;
    }
  }
  a.S = best_S;
  return launch_kernel(kern, dim3((unsigned)(tiles * best_S)), dim3(kWrThreads), smem, st,
                       (unsigned)best_S, m, a);
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
  a.NE = (E + 31) / 32 * 32;
  a.nbc = (E + 63) / 64;
  a.kb_total = (T + 63) / 64;
  a.stage_bytes = 2 * kChunk + 2 * a.nbc * kChunk;
  a.ps = a.NE + 4;
  const int extra = (kWrConv * 8 + 256) * 4 + (2 * kWrMaxStages + 1) * 8 + 16;
  const int room = 227 * 1024 - 1024 - extra;
  a.stages = room / a.stage_bytes;
  if (a.stages > kWrMaxStages) a.stages = kWrMaxStages;
  if (a.stages < 2 || a.stages * a.stage_bytes < 128 * a.ps * 4) return MOE_OK;
  const int tiles = (d + 127) / 128;
  a.S = 1;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  const size_t smem = (size_t)(1024 + a.stages * a.stage_bytes + extra);
  launch_begin(K_ROUTER_DWR, st);
  cudaError_t e;
  switch (a.nbc) {
    case 1: e = launch_dwr<8>(tiles, smem, st, mx, a); break;
    case 2: e = launch_dwr<16>(tiles, smem, st, mx, a); break;
    case 3: e = launch_dwr<24>(tiles, smem, st, mx, a); break;
    default: e = launch_dwr<32>(tiles, smem, st, mx, a); break;
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
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
