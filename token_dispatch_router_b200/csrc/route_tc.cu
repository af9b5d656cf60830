// Router on the tensor cores for bf16 shapes: logits = x W_r (+ bias) with tcgen05, then
// softmax and top-K in the epilogue.
//
// "How AI chips support MoE", chapter 4, section 4.2: the gate is a small dense linear map
// that every token passes through and that the experts wait on; section 4.3: top-K is a
// partial sort per token. "Two upstream innovations of MoE: Routing-Free and OmniMoE",
// section 1.1: Router -> Softmax -> TopK.
//
// The product is computed transposed, D[e, t] = sum_k W_r[k, e] x[t, k]: experts on the
// MMA's M (one 128-row M tile per 128 experts; rows past E are never read) and tokens on its
// N (up to 256 per instruction). The router's contraction d is long and its output narrow,
// so the kernel's cost is the number of tcgen05.mma instructions one thread issues per CTA,
// (d / S / 16) per M tile, not their size: putting 256 tokens on N instead of 128 on M
// halves that count, and an instruction of N = 256 costs the tensor pipe no more than the
// issue loop sustains.
// Layout: one tile of up to 256 tokens per cluster of S CTAs (S = 1, 2, 4 or 8) that split
// the d contraction into contiguous ranges of 64-wide k-blocks. Operands: A = W_r rows
// [64 k][64 e] as MN-major 128-byte-swizzled chunks (one TMA box per chunk, experts past E
// zero-filled); B = the x tile [rows][64 k], K-major, 128-byte swizzle. The partial
// D[e, t] (fp32, TMEM lanes = experts, columns = tokens) is copied to shared memory as
// [e][t] rows; after a cluster barrier every rank finishes a contiguous share of the tile's
// tokens, G threads per token (each owning experts g, g + G, ...), adding the partials of
// ranks 0..S-1 in that order through distributed shared memory (deterministic: the same
// fp32 sum in the same order whichever rank does it), + bias, optional logits store, a
// register top-KM list per thread (value descending, ties to the lower id, +0 == -0), the G
// lists merged by a bitonic network over shuffles, softmax weights over the selected
// (renormalised) or over all E (online sum, merged the same way).
// Roles (256 threads): warp 0 issues the TMA loads, warp 1 the MMAs, both as warp-uniform
// loops with one elected lane issuing; warps 4m..4m+3 read M tile m from TMEM (warp w owns
// lanes 32 (w % 4) ...); all eight warps reduce. Each tile starts its k-blocks at a
// different offset so that the CTAs do not all read the same W_r lines at once.
// Every mbarrier wait is bounded; on expiry the status word records MOE_ERR_TIMEOUT and the
// CTA skips its remaining work (cluster barriers are still passed, so no peer waits).
#include <math.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "topk.cuh"

namespace moe {

namespace {

using namespace ptx;

constexpr int RBK = 64;                  // k per stage: one 128-byte swizzle atom of bf16
constexpr int RCHUNK = RBK * 64 * 2;     // 8 KB: A chunk of 64 k-rows x 64 experts
constexpr int R_THREADS = 256;
constexpr int KMAX = 8;
constexpr int R_SMEM_MAX = 227 * 1024;
constexpr int R_MAX_STAGES = 8;

struct RouteArgs {
  const float* bias;
  float* logits_out;
  int32_t* topk_ids;
  float* topk_w;
  int T, E, K, renorm;
  int kblocks;   // d / 64
  int S;         // CTAs of a cluster splitting d
  int rows;      // tokens per tile (<= 256); tile i holds tokens [i rows, (i + 1) rows)
  int nmma;      // the MMA's N: rows rounded up to 16
  int a_chunks;  // W_r chunks loaded per stage: ceil(E / 64)
  int a_slot;    // bytes of a stage's A slot: 16 KB per M tile
  int stage_bytes, stages, tx_bytes, bar_off;
  int ps;        // row stride (floats) of the partial tile part[e][t] in shared memory
  int G;         // threads per token in the epilogue (1, 2, 4 or 8)
  int vec_logits;  // G == 1 and logits_out 16-byte aligned: rows stored as float4
  unsigned* status;
  unsigned long long limit_ns;
};

__device__ __forceinline__ uint32_t elect_one() {
  uint32_t p = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 R;\n\telect.sync R|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}\n"
      : "=r"(p));
  return p;
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Eight of one token's experts, e = e0 + G j: their partials from every rank (loaded first,
// S x 8 loads in flight, at addresses clamped into the tile so that no load sits behind a
// branch), added in rank order, + bias, into the thread's top-K list and plain-softmax sums,
// and stored as logits. FULL: all eight experts exist (no per-expert checks).
template <int KM, int S, bool FULL>
__device__ __forceinline__ void route_batch(float (&bv)[KM], int (&be)[KM], float& mx, float& ssum,
                                            const uint32_t (&rbase)[S], uint32_t colb, int e0,
                                            const RouteArgs& g, float* lrow) {
  const int E = g.E, G = g.G;
  float pv[S][8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = FULL ? e0 + G * j : min(e0 + G * j, E - 1);
    const uint32_t off = colb + (uint32_t)(e * g.ps * 4);
#pragma unroll
    for (int q = 0; q < S; ++q)
      pv[q][j] = S > 1 ? ld_dsmem_f32(rbase[q] + off) : ld_shared_f32(rbase[q] + off);
  }
  float lv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float l = pv[0][j];
#pragma unroll
    for (int q = 1; q < S; ++q) l += pv[q][j];
    const int e = e0 + G * j;
    if (g.bias != nullptr) l += g.bias[FULL ? e : min(e, E - 1)];
    lv[j] = l;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = e0 + G * j;
    if (FULL || e < E) {
      top_insert<KM>(bv, be, lv[j], e);
      if (!g.renorm) {
        if (lv[j] > mx) {
          ssum = ssum * expf(mx - lv[j]) + 1.f;
          mx = lv[j];
        } else {
          ssum += expf(lv[j] - mx);
        }
      }
    }
  }
  if (lrow != nullptr) {
    if (FULL && G == 1 && g.vec_logits) {  // e = e0 + j: two whole float4 groups
      *reinterpret_cast<float4*>(lrow + e0) = make_float4(lv[0], lv[1], lv[2], lv[3]);
      *reinterpret_cast<float4*>(lrow + e0 + 4) = make_float4(lv[4], lv[5], lv[6], lv[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (FULL || e0 + G * j < E) lrow[e0 + G * j] = lv[j];
    }
  }
}

// MT: M tiles of 128 experts (1 or 2); KM >= K, a power of two <= 8; S: CTAs of a cluster
// splitting d (1, 2, 4 or 8).
template <int MT, int KM, int S>
__global__ void __launch_bounds__(R_THREADS, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const RouteArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  const int RSTAGES = g.stages, STAGE = g.stage_bytes, A_SLOT = g.a_slot;
  uint64_t* bars = (uint64_t*)(base + g.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + RSTAGES;
  uint64_t* accf = bars + 2 * RSTAGES;
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * RSTAGES + 1);
  constexpr uint32_t TCOLS = MT == 1 ? 256 : 512;  // accumulator m at column 256 m

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = S > 1 ? cluster_rank() : 0u;
  const int tile = S > 1 ? (int)cluster_id_x() : (int)blockIdx.x;
  const int kb0 = (int)(rank * g.kblocks / S), kb1 = (int)((rank + 1) * g.kblocks / S);
  const int nkb = kb1 - kb0, rot = nkb > 0 ? tile % nkb : 0;

  if (tid == 32) {  // fetch both tensor maps while the barriers are set up
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < RSTAGES; ++s) {
      mbar_init(saddr(&full[s]), 1);
      mbar_init(saddr(&empty[s]), 1);
    }
    mbar_init(saddr(accf), 1);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();

  // The producer starts loading at once; the MMA warp allocates the accumulators meanwhile.
  if (warp == 0) {
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      const int kb = kb0 + (i + rot) % nkb;
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&empty[stage]), phase ^ 1u, nullptr, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      if (elect_one()) {
        const uint32_t fb = saddr(&full[stage]);
        mbar_expect_tx(fb, (uint32_t)g.tx_bytes);
        const uint32_t a = saddr(ring + stage * STAGE);
        tma_load_2d(a + A_SLOT, &tmX, kb * RBK, tile * g.rows, fb);
        for (int c = 0; c < g.a_chunks; ++c) tma_load_2d(a + c * RCHUNK, &tmW, c * 64, kb * RBK, fb);
      }
      __syncwarp();
      if (++stage == RSTAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  } else if (warp == 1) {
    tmem_alloc<1>(saddr(tmem_slot), TCOLS);
    tc_fence_before();
    __syncwarp();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Descriptors of stage 0; a stage (and a 16-wide k step) moves the start-address field,
    // which holds shared-memory byte addresses / 16 (below 2^14, so adding does not carry).
    // A (MN-major): 64-expert chunks 8 KB apart, 8-row k groups 1 KB apart, a k step = 16
    // rows = 2 KB. B (K-major): 128-byte rows, 8-row groups 1 KB apart, a k step = 32 bytes.
    const uint64_t ad0 = desc_sw128(saddr(ring), RCHUNK, 1024);
    const uint64_t bd0 = desc_sw128(saddr(ring) + A_SLOT, 16, 1024);
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                           ((uint32_t)(g.nmma >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    int stage = 0;
    uint32_t phase = 0;
    for (int i = 0; i < nkb; ++i) {
      int w = 0;
      if (lane == 0) w = mbar_wait(saddr(&full[stage]), phase, nullptr, g.status, g.limit_ns);
      if (!__shfl_sync(0xffffffffu, w, 0)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t so = (uint64_t)((stage * STAGE) >> 4);
#pragma unroll
        for (int kk = 0; kk < RBK / 16; ++kk) {
#pragma unroll
          for (int m = 0; m < MT; ++m)
            tc_mma<1>(tmem + (uint32_t)(256 * m),
                      ad0 + so + (uint64_t)(m * (2 * RCHUNK >> 4) + kk * 128),
                      bd0 + so + (uint64_t)(kk * 2), idesc, (i | kk) != 0 ? 1u : 0u);
        }
        tc_commit<1>(saddr(&empty[stage]));
      }
      __syncwarp();
      if (++stage == RSTAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (elect_one()) tc_commit<1>(saddr(accf));
  }
  __syncwarp();

  // ---- the partial tile to shared memory: part[e][t], e < E, t < nmma (row stride ps)
  int w_ok = 0;
  if (lane == 0) w_ok = mbar_wait(saddr(accf), 0, nullptr, g.status, g.limit_ns);
  w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
  tc_fence_before();
  __syncthreads();  // the ring is free (every MMA has completed); the TMEM address is set
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool have = w_ok && nkb > 0;  // this CTA accumulated a partial
  const uint32_t part = saddr(ring);
  {
    // warp w reads TMEM lanes 32 (w % 4) ...; with one M tile, warps w and w + 4 take
    // alternate 64-column blocks of the same lanes; four 16-column loads, then one wait
    const int q = warp & 3;
    const int m = MT == 1 ? 0 : warp >> 2;
    const int c_first = MT == 1 ? 64 * (warp >> 2) : 0, c_step = MT == 1 ? 128 : 64;
    const int e = 128 * m + 32 * q + lane;
    if (128 * m + 32 * q < g.E) {  // warp-uniform: this warp holds experts
      const uint32_t trow = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(256 * m);
      for (int c0 = c_first; c0 < g.nmma; c0 += c_step) {
        uint32_t v[4][16];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          if (c0 + 16 * h < g.nmma) tmem_ld16(trow + (uint32_t)(c0 + 16 * h), v[h]);
        tmem_ld_wait();
        if (e < g.E) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            if (c0 + 16 * h < g.nmma) {
              const uint32_t dst = part + (uint32_t)((e * g.ps + c0 + 16 * h) * 4);
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                st_shared_v4(dst + j * 4, have ? __uint_as_float(v[h][j]) : 0.f,
                             have ? __uint_as_float(v[h][j + 1]) : 0.f,
                             have ? __uint_as_float(v[h][j + 2]) : 0.f,
                             have ? __uint_as_float(v[h][j + 3]) : 0.f);
            }
          }
        }
      }
    }
  }
  if (S > 1)
    cluster_sync();  // every rank's partial is in its shared memory
  else
    __syncthreads();

  // ---- this rank's share of the tile's tokens: G threads per token (thread gi owns experts
  // gi, gi + G, ...), R_THREADS / G tokens a pass
  const int E = g.E, K = g.K, G = g.G;
  const int share = (g.rows + S - 1) / S;
  const int tl = tid / G, gi = tid % G;
  uint32_t rbase[S];  // the partial tile of each rank, in the cluster's shared window
#pragma unroll
  for (int q = 0; q < S; ++q) rbase[q] = S > 1 ? map_rank(part, (uint32_t)q) : part;
  const bool whole = E % (8 * G) == 0;  // every batch of eight experts is whole
  for (int p0 = 0; p0 < share; p0 += R_THREADS / G) {
    const int col = (int)rank * share + p0 + tl;  // token column inside the tile
    const int t = tile * g.rows + col;
    const bool mine = p0 + tl < share && col < g.rows && t < g.T;
    float bv[KM];
    int be[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      bv[k] = -INFINITY;
      be[k] = -1;
    }
    float mx = -INFINITY, ssum = 0.f;  // online max / sum of exp for the plain softmax
    if (mine) {
      float* lrow = g.logits_out != nullptr ? g.logits_out + (size_t)t * E : nullptr;
#pragma unroll 1
      for (int e0 = gi; e0 < E; e0 += 8 * G) {  // eight of this thread's experts at a time
        if (whole)
          route_batch<KM, S, true>(bv, be, mx, ssum, rbase, (uint32_t)(col * 4), e0, g, lrow);
        else
          route_batch<KM, S, false>(bv, be, mx, ssum, rbase, (uint32_t)(col * 4), e0, g, lrow);
      }
    }
    // merge the G lists of a token (lanes G tl .. G tl + G - 1 of one warp)
    for (int h = 1; h < G; h <<= 1) {
      top_merge<KM>(bv, be, h);
      if (!g.renorm) {
        const float om = __shfl_xor_sync(0xffffffffu, mx, h);
        const float os = __shfl_xor_sync(0xffffffffu, ssum, h);
        const float nm = fmaxf(mx, om);
        if (nm != -INFINITY) {
          ssum = (mx == -INFINITY ? 0.f : ssum * expf(mx - nm)) +
                 (om == -INFINITY ? 0.f : os * expf(om - nm));
          mx = nm;
        }
      }
    }
    if (mine && gi == 0) {
      const float top = bv[0];
      float den = 0.f;
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k < K) den += expf(bv[k] - top);
      if (!g.renorm) den = ssum * expf(mx - top);
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (k < K) {
          g.topk_ids[(size_t)t * K + k] = be[k];
          g.topk_w[(size_t)t * K + k] = expf(bv[k] - top) / den;
        }
      }
    }
  }
  if (S > 1) {
    // This rank's reads of its peers' partials are done (their values are in registers): a
    // relaxed arrive, so that it does not wait for this thread's global stores; then no CTA
    // exits while a peer may still read its partial.
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    cluster_wait();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, TCOLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box0,
                 uint32_t box1) {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = (EncodeTiledFn)p;
  }
  cuuint64_t gd[2] = {inner, outer}, gs[1] = {inner * 2};
  cuuint32_t bx[2] = {box0, box1}, es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stage layout for `rows` tokens: A slot (16 KB per M tile) then the x tile (nmma rows of
// 128 B); as many stages as fit, at most R_MAX_STAGES; the partial tile [E][ps] must fit in
// the ring. Returns the dynamic shared memory size, or 0 if it does not fit.
int ring_layout(int MT, int E, int rows, RouteArgs& a) {
  a.nmma = ((rows + 15) / 16) * 16;
  a.a_chunks = (E + 63) / 64;
  a.a_slot = MT * 2 * RCHUNK;
  a.stage_bytes = a.a_slot + a.nmma * 128;
  a.tx_bytes = a.a_chunks * RCHUNK + rows * 128;
  a.ps = a.nmma + 4;  // v4 stores of 32 lanes land on 8 distinct bank groups
  auto smem_of = [&](int st) { return 1024 + st * a.stage_bytes + (2 * st + 2) * 8; };
  int st = R_MAX_STAGES;
  while (st > 2 && smem_of(st) > R_SMEM_MAX) --st;
  a.stages = st;
  a.bar_off = st * a.stage_bytes;
  if (smem_of(st) > R_SMEM_MAX || E * a.ps * 4 > a.bar_off) return 0;
  return smem_of(st);
}

// Clusters of S CTAs of `kern` that can be resident at once (clusters stay inside one GPC,
// so this can be below SMs / S); cached per device, kernel, S and shared-memory size.
int active_clusters(const void* kern, int smem, int S) {
  struct Entry {
    const void* kern;
    int dev, S, smem, n;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].kern == kern && cache[i].dev == dev && cache[i].S == S && cache[i].smem == smem)
      return cache[i].n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S);
  cfg.blockDim = dim3(R_THREADS);
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
  if (used < 64) cache[used++] = Entry{kern, dev, S, smem, n};
  return n;
}

template <int MT, int KM, int S>
const void* kernel_for() {
  return (const void*)route_tc_kernel<MT, KM, S>;
}

template <int MT, int KM, int S>
moe_status launch_cfg(const moe_shape& s, const void* x, const void* w_r, const RouteArgs& a,
                      int tiles, int smem, cudaStream_t st) {
  auto kern = route_tc_kernel<MT, KM, S>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, R_SMEM_MAX) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  CUtensorMap mx, mw;
  if (!make_map_2d(&mx, x, (uint64_t)(a.kblocks * RBK), (uint64_t)s.T, 64, (uint32_t)a.rows))
    return MOE_ERR_CUDA;
  if (!make_map_2d(&mw, w_r, (uint64_t)s.E, (uint64_t)(a.kblocks * RBK), 64, 64))
    return MOE_ERR_CUDA;
  launch_begin(K_ROUTE_TC, st);
  launch_kernel(kern, dim3((unsigned)(tiles * S)), dim3(R_THREADS), (size_t)smem, st,
                (unsigned)S, mx, mw, a);
  return launch_end(K_ROUTE_TC, st);
}

template <int MT, int KM>
moe_status launch_mk(const moe_shape& s, const void* x, const void* w_r, RouteArgs a,
                     cudaStream_t st) {
  // Tiles of up to 256 tokens (fewer when E * (rows + 4) floats would not fit the ring).
  int max_rows = 256;
  RouteArgs probe = a;
  while (max_rows > 16 && ring_layout(MT, s.E, max_rows, probe) == 0) max_rows -= 16;
  const int smem_max = ring_layout(MT, s.E, max_rows, probe);
  if (smem_max == 0) return MOE_ERR_UNSUPPORTED;
  // Split d over the largest S in {8, 4, 2, 1} (each rank keeping at least two k-blocks)
  // whose clusters, all resident at once, hold every 256-token tile; then shorten the tiles
  // so that the resident clusters are all used (at least 16 tokens a tile).
  const void* kern_s[4] = {kernel_for<MT, KM, 1>(), kernel_for<MT, KM, 2>(),
                           kernel_for<MT, KM, 4>(), kernel_for<MT, KM, 8>()};
  const int tiles0 = (s.T + max_rows - 1) / max_rows;
  int S = 1, fit = sm_count();
  for (int si = 3; si >= 1; --si) {
    const int cand = 1 << si;
    if (2 * cand > a.kblocks) continue;
    if (cudaFuncSetAttribute(kern_s[si], cudaFuncAttributeMaxDynamicSharedMemorySize,
                             R_SMEM_MAX) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int f = active_clusters(kern_s[si], smem_max, cand);
    if (f >= tiles0) {
      S = cand;
      fit = f;
      break;
    }
  }
  int tiles = fit;
  if (tiles < tiles0) tiles = tiles0;
  if (tiles > (s.T + 15) / 16) tiles = (s.T + 15) / 16;
  a.rows = (s.T + tiles - 1) / tiles;
  if (a.rows > max_rows) a.rows = max_rows;
  tiles = (s.T + a.rows - 1) / a.rows;
  a.S = S;
  const int smem = ring_layout(MT, s.E, a.rows, a);
  if (smem == 0) return MOE_ERR_UNSUPPORTED;
  // Threads per token: one up to 32 experts, then enough for about 32 experts each (their
  // top-K lists merged by shuffles).
  int G = 1;
  while (G < 8 && 32 * G < s.E) G *= 2;
  a.G = G;
  a.vec_logits = G == 1 && ((uintptr_t)a.logits_out & 15) == 0;
  switch (S) {
    case 8: return launch_cfg<MT, KM, 8>(s, x, w_r, a, tiles, smem, st);
    case 4: return launch_cfg<MT, KM, 4>(s, x, w_r, a, tiles, smem, st);
    case 2: return launch_cfg<MT, KM, 2>(s, x, w_r, a, tiles, smem, st);
    default: return launch_cfg<MT, KM, 1>(s, x, w_r, a, tiles, smem, st);
  }
}

template <int MT>
moe_status launch_m(const moe_shape& s, const void* x, const void* w_r, const RouteArgs& a,
                    cudaStream_t st) {
  if (s.K <= 2) return launch_mk<MT, 2>(s, x, w_r, a, st);
  if (s.K <= 4) return launch_mk<MT, 4>(s, x, w_r, a, st);
  return launch_mk<MT, 8>(s, x, w_r, a, st);
}

}  // namespace

bool route_tc_supported(const moe_shape& s) {
  return s.dtype == MOE_BF16 && s.E % 8 == 0 && s.E <= 256 && s.K <= KMAX && s.d % 64 == 0;
}

moe_status launch_route_tc(const moe_shape& s, const void* x, const void* w_r, const float* bias,
                           float* logits_out, int32_t* ids, float* w, cudaStream_t st) {
  RouteArgs a = {};
  a.bias = bias;
  a.logits_out = logits_out;
  a.topk_ids = ids;
  a.topk_w = w;
  a.T = s.T;
  a.E = s.E;
  a.K = s.K;
  a.renorm = s.renormalize;
  a.kblocks = s.d / RBK;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  if (s.E <= 128) return launch_m<1>(s, x, w_r, a, st);
  return launch_m<2>(s, x, w_r, a, st);
}

}  // namespace moe
