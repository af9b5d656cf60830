// bf16 grouped SwiGLU FFN on the 5th-generation tensor cores (tcgen05 + TMEM, fed by TMA).
//
// SonicMoE explainer (gitcode.csdn.net):
//   section 3 items 3-5 - grouped GEMM whose M differs per expert, SwiGLU, second GEMM;
//   section 6.2         - gather fusion: the GEMM reads the rows of x by routing index
//                         while loading its operand, so no [T*K, d] gathered copy exists;
//   section 6.3         - epilogue fusion: SwiGLU is applied while the accumulator is on
//                         chip (here in TMEM) before anything goes back to HBM.
//
// One persistent kernel per GEMM (grid = #SMs, one CTA per SM), warp-specialised:
//   warp 0     TMA producer: the B tile 64 x 256 bf16 as four 64 x 64 boxes of the
//              expert's weights (and, for the down GEMM, the A tile: one tiled load of
//              128 a_act rows) into a 4-stage shared-memory ring (48 KB a stage, 128-byte
//              swizzle) signalled through mbarrier transaction counts;
//   warps 6-9  (gate/up only) the gathered A tile 128 x 64 bf16: each lane copies 16-byte
//              pieces of x rows, row = perm_to_assign[p] / K, with cp.async straight into
//              the 128-byte-swizzled layout the MMA descriptor expects, and signals the
//              stage with cp.async.mbarrier.arrive.noinc. Eight lanes cover one 128-byte
//              row segment, so each warp instruction moves four whole segments. (The
//              tensor-map gather4 form measured 2.6x slower here: 128 row requests per
//              stage starve the tensor pipe.)
//   warp 1     TMEM allocator and MMA issuer: one thread issues tcgen05.mma (M=128,
//              N=256, K=16, bf16 in, fp32 accumulate) four times per stage and commits
//              each stage back to the producer; two 256-column accumulators in TMEM
//              (all 512 columns) let the epilogue of one tile overlap the next tile;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one output row
//              per thread), gate/up: silu(g) * u -> bf16 a_act; down: bf16 y_perm.
// Gate/up tile: accumulator columns [0,128) = W_gate columns n0..n0+127 and [128,256) =
// W_up columns n0..n0+127, so SwiGLU pairs lie in one thread's registers.
// Work order: expert-major, then N-tile, with the M-tiles of an expert fastest, so the
// CTAs running at one time share each expert's weight panel through L2.
// The variable-M tile table is built on the device from offsets[] by every CTA: no host
// sync. Every mbarrier wait is bounded (kWaitLimitNs); on expiry the CTA records
// MOE_ERR_TIMEOUT, stops issuing, waits (bounded) for its copies and MMAs in flight,
// frees its TMEM and returns.
#include "ffn_args.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BK = 64, BN = 256, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;           // 16 KB
constexpr int B_CHUNK = BK * 64 * 2;           // one 64 x 64 bf16 box, 8 KB
constexpr int B_BYTES = 4 * B_CHUNK;           // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS_DOWN = 192;   // producer, MMA, 4 epilogue warps
constexpr int THREADS_GATEUP = 320; // + 4 gather warps
constexpr int GATHER_WARP0 = 6;
constexpr int GATHER_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAXE = 256;
constexpr int SMEM_TAIL = 4096;  // barriers, TMEM slot, abort flag, tile table
// epilogue staging: per epilogue warp, its 32 rows of one 32-column output chunk, rows
// padded to 80 bytes so that a thread writing its own row hits distinct banks
constexpr int EPI_ROW = 80;
constexpr int EPI_WARP_BYTES = 32 * EPI_ROW;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + SMEM_TAIL + 4 * EPI_WARP_BYTES;

// Instruction descriptor, kind::f16: D fp32 (bit 4), A bf16 (bits 7-9 = 1), B bf16
// (bits 10-12 = 1), A K-major (bit 15 = 0), B MN-major (bit 16 = 1), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);


// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: true once the phase of `parity` completed; false on abort or timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          const GemmArgs& g, uint64_t limit) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit) {
      report(g.status, MOE_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
// 16 bytes global -> shared, cached in L2 only; completion tracked per thread.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(dst), "l"(src)
               : "memory");
}
// The barrier receives one arrival once every cp.async this thread issued so far landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1 (bit 46).
// K-major operand (A): rows of 128 B, 8-row groups 1024 B apart (SBO); LBO unused (16).
// MN-major operand (B): 64-element MN chunks LBO bytes apart, 8-row K groups SBO apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

struct Tile {
  int e, m0, rows, n0;
};

__device__ __forceinline__ Tile decode_tile(int w, const int* s_off, const int* s_cum,
                                            const int* s_mt, int E, int out_tile) {
  int lo = 0, hi = E - 1;  // largest e with s_cum[e] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_cum[mid] <= w) lo = mid;
    else hi = mid - 1;
  }
  Tile t;
  t.e = lo;
  const int local = w - s_cum[lo];
  const int mt = s_mt[lo];
  const int m = local % mt;
  t.n0 = (local / mt) * out_tile;
  t.m0 = s_off[lo] + m * BM;
  t.rows = min(BM, s_off[lo + 1] - t.m0);
  return t;
}

template <bool GATEUP>
__global__ void __launch_bounds__(GATEUP ? THREADS_GATEUP : THREADS_DOWN, 1)
    grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = base;
  uint64_t* bars = (uint64_t*)(base + STAGES * STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint64_t* done = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 5);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* s_off = (int*)(tmem_slot + 2);
  int* s_cum = s_off + MAXE + 1;
  int* s_mt = s_cum + MAXE + 1;
  uint8_t* epi = base + STAGES * STAGE_BYTES + SMEM_TAIL;  // epilogue staging (16-byte aligned)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = g.E;
  constexpr int NTHREADS = GATEUP ? THREADS_GATEUP : THREADS_DOWN;
  // full[s]: the TMA thread's expect_tx arrival (+ one noinc arrival per gather thread)
  constexpr uint32_t FULL_COUNT = GATEUP ? 1 + GATHER_THREADS : 1;
  constexpr uint32_t TMA_BYTES = GATEUP ? B_BYTES : STAGE_BYTES;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(saddr(&full[s]), FULL_COUNT);
      mbar_init(saddr(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&tfull[b]), 1);
      mbar_init(saddr(&tempty[b]), 128);
    }
    mbar_init(saddr(done), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  for (int i = tid; i <= E; i += NTHREADS) s_off[i] = g.offsets[i];
  __syncthreads();
  if (warp == 0) {  // tile table: s_mt[e] = ceil(kept_e / BM); s_cum = n_tiles * prefix
    constexpr int PER = MAXE / 32;
    int loc[PER], sum = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      loc[j] = (e < E) ? (s_off[e + 1] - s_off[e] + BM - 1) / BM : 0;
      sum += loc[j];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      if (e < E) {
        s_mt[e] = loc[j];
        s_cum[e] = run * g.n_tiles;
      }
      run += loc[j];
    }
    if (lane == 31) s_cum[E] = incl * g.n_tiles;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_cum[E];
  const uint64_t limit = g.limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;  // per stage: ever issued, parity of last issue
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Tile t = decode_tile(w, s_off, s_cum, s_mt, E, g.out_tile);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0) w_ok = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g, limit);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const uint32_t fb = saddr(&full[stage]);
        if (lane == 0) mbar_expect_tx(fb, TMA_BYTES);
        __syncwarp();
        const uint32_t a_dst = saddr(ring + stage * STAGE_BYTES);
        const uint32_t b_dst = a_dst + A_BYTES;
        if (!GATEUP && lane == 0) tma_load_2d(a_dst, &tmA, kb * BK, t.m0, fb);
        if (lane < 4) {
          if (GATEUP) {
            const CUtensorMap* mp = (lane < 2) ? &tmB0 : &tmB1;
            tma_load_3d(b_dst + lane * B_CHUNK, mp, t.n0 + (lane & 1) * 64, kb * BK, t.e, fb);
          } else {
            tma_load_3d(b_dst + lane * B_CHUNK, &tmB0, t.n0 + lane * 64, kb * BK, t.e, fb);
          }
        }
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
    }
    // Drain: the last load issued into each stage has landed (bounded).
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) {
        if (!(issued_mask & (1u << s))) continue;
        const uint32_t par = (issued_par >> s) & 1u;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try(saddr(&full[s]), par) && globaltimer_ns() - t0 < limit) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(saddr(&tempty[buf]), (use & 1u) ^ 1u, abort_flag, g, limit)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(saddr(&full[stage]), phase, abort_flag, g, limit)) {
            ok = false;
            break;
          }
          if (GATEUP) fence_proxy_async_smem();  // cp.async (generic) writes -> MMA reads
          tc_fence_after();
          const uint32_t a_addr = saddr(ring + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = desc_sw128(b_addr + kk * 2048, B_CHUNK, 1024);
            tc_mma(d_tmem, ad, bd, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit(saddr(&empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit(saddr(&tfull[buf]));
      }
      // every MMA this thread issued has completed before TMEM is released (bounded)
      tc_commit(saddr(done));
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try(saddr(done), 0) && globaltimer_ns() - t0 < limit) {
      }
    }
  } else if (GATEUP && warp >= GATHER_WARP0) {
    // ------------------------------------------------------------ A gather (warps 6-9)
    const int gw = warp - GATHER_WARP0;  // rows [32 gw, 32 gw + 32)
    const int c = lane & 7;              // 16-byte piece of the 128-byte row segment
    const int rg = lane >> 3;            // rows 32 gw + rg + 4 i, i < 8
    int stage = 0;
    uint32_t phase = 0;
    // token rows of a tile: row r of the tile reads x[perm_to_assign[m0 + r] / K]
    auto rows_of = [&](int w, const uint8_t* (&src)[8]) {
      const Tile t = decode_tile(w, s_off, s_cum, s_mt, E, g.out_tile);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = gw * 32 + rg + 4 * i;
        const int p = t.m0 + (r < t.rows ? r : 0);  // padding rows reuse the tile's first row
        const int a = g.p2a[p];
        int tk = a / g.K;
        if (a < 0 || tk >= g.T) {
          report(g.status, MOE_ERR_DEVICE_INDEX);
          tk = 0;
        }
        src[i] = g.x + (size_t)tk * g.x_row_bytes + c * 16;
      }
    };
    uint32_t dst[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = gw * 32 + rg + 4 * i;
      dst[i] = (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));  // 128-byte swizzle
    }
    const uint8_t* src[8];
    if (blockIdx.x < (unsigned)total) rows_of(blockIdx.x, src);
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      // the next tile's rows are loaded now, one tile ahead of their use
      const uint8_t* nsrc[8];
      if (w + (int)gridDim.x < total) rows_of(w + gridDim.x, nsrc);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0) w_ok = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g, limit);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        const uint32_t a_dst = saddr(ring + stage * STAGE_BYTES);
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16(a_dst + dst[i], src[i] + (size_t)kb * (BK * 2));
        cp_async_arrive_noinc(saddr(&full[stage]));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int i = 0; i < 8; ++i) src[i] = nsrc[i];
    }
    cp_async_wait_all();  // nothing of ours lands after the CTA exits
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 are reachable from this warp
    const int r = q * 32 + lane;
    int it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      const Tile t = decode_tile(w, s_off, s_cum, s_mt, E, g.out_tile);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      int w_ok = 0;
      if (lane == 0) w_ok = mbar_wait(saddr(&tfull[buf]), use & 1u, abort_flag, g, limit);
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t)(buf * BN) + ((uint32_t)(q * 32) << 16);
      const bool row_ok = r < t.rows;
      bf16* orow = g.out + (size_t)(t.m0 + (row_ok ? r : 0)) * g.ld_out;
      if (GATEUP) {
        // each thread computes its row's 32 columns of a chunk; the warp's 32 rows go out
        // through its padded buffer, one instruction storing 8 whole 64-byte row segments
        uint8_t* ebuf = epi + q * EPI_WARP_BYTES;
        const int lr = lane >> 2, lc = lane & 3;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tb + c * 32, gv);
          tmem_ld32(tb + 128 + c * 32, uv);
          tmem_ld_wait();
          const int col = t.n0 + c * 32;
          {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g0 = __uint_as_float(gv[2 * j]), g1 = __uint_as_float(gv[2 * j + 1]);
              const float u0 = __uint_as_float(uv[2 * j]), u1 = __uint_as_float(uv[2 * j + 1]);
              const float h0 = __fdividef(g0, 1.f + __expf(-g0)) * u0;
              const float h1 = __fdividef(g1, 1.f + __expf(-g1)) * u1;
              pk[j] = pack_bf16x2(h0, h1);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<uint4*>(ebuf + lane * EPI_ROW + j * 16) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
          __syncwarp();
          if (col < g.n_out) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rr = q * 32 + lr + 8 * i;
              if (rr < t.rows)
                *reinterpret_cast<uint4*>(g.out + (size_t)(t.m0 + rr) * g.ld_out + col + lc * 8) =
                    *reinterpret_cast<const uint4*>(ebuf + (lr + 8 * i) * EPI_ROW + lc * 16);
            }
          }
          __syncwarp();  // the buffer is free for the next chunk
          if (row_ok && col < g.n_out && g.h_out != nullptr) {  // keep (g | u) for the backward
            bf16* hrow = g.h_out + (size_t)(t.m0 + r) * (2 * (size_t)g.n_out);
            uint4* hg = reinterpret_cast<uint4*>(hrow + col);
            uint4* hu = reinterpret_cast<uint4*>(hrow + g.n_out + col);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              hg[j] = make_uint4(pack_bf16x2(__uint_as_float(gv[8 * j]), __uint_as_float(gv[8 * j + 1])),
                                 pack_bf16x2(__uint_as_float(gv[8 * j + 2]), __uint_as_float(gv[8 * j + 3])),
                                 pack_bf16x2(__uint_as_float(gv[8 * j + 4]), __uint_as_float(gv[8 * j + 5])),
                                 pack_bf16x2(__uint_as_float(gv[8 * j + 6]), __uint_as_float(gv[8 * j + 7])));
              hu[j] = make_uint4(pack_bf16x2(__uint_as_float(uv[8 * j]), __uint_as_float(uv[8 * j + 1])),
                                 pack_bf16x2(__uint_as_float(uv[8 * j + 2]), __uint_as_float(uv[8 * j + 3])),
                                 pack_bf16x2(__uint_as_float(uv[8 * j + 4]), __uint_as_float(uv[8 * j + 5])),
                                 pack_bf16x2(__uint_as_float(uv[8 * j + 6]), __uint_as_float(uv[8 * j + 7])));
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + c * 32, v);
          tmem_ld_wait();
          const int col = t.n0 + c * 32;
          if (row_ok && col < g.n_out) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(saddr(&tempty[buf]));
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace

// ------------------------------------------------------------------ host: tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(ptr), gd, gs,
            bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <bool GATEUP>
moe_status run_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                    const GemmArgs& args, cudaStream_t st, int kid) {
  auto kern = grouped_gemm_tc<GATEUP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  launch_begin(kid, st);
  launch_kernel(kern, dim3((unsigned)sm_count()), dim3(GATEUP ? THREADS_GATEUP : THREADS_DOWN),
                SMEM_BYTES, st, 1, a, b0, b1, args);
  return launch_end(kid, st);
}

// Failure-detection self test: waits on an mbarrier that nothing completes; the bounded
// wait gives up after limit_ns, records MOE_ERR_TIMEOUT and the kernel returns.
__global__ void selftest_timeout_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(saddr(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    GemmArgs g;
    g.status = status;
    mbar_wait(saddr(&bar), 0, &abort_flag, g, limit_ns);
    mbar_arrive(saddr(&bar));  // complete the phase so the barrier is left idle
  }
  __syncthreads();
}

}  // namespace

moe_status launch_selftest_timeout(uint64_t limit_ns, cudaStream_t st) {
  launch_begin(K_SELFTEST, st);
  selftest_timeout_kernel<<<1, 32, 0, st>>>(device_status_ptr(), limit_ns);
  return launch_end(K_SELFTEST, st);
}

// Tensor maps and arguments of both GEMMs for one call.
struct FfnMaps {
  CUtensorMap mg, mu, ma, md;
  GemmArgs gate_up, down;
};

static moe_status prepare_ffn(const moe_shape& s, const void* x, const int32_t* offsets,
                              const int32_t* p2a, const void* w_gate, const void* w_up,
                              const void* w_down, void* a_act, void* y_perm, FfnMaps& f) {
  const uint64_t d = s.d, n = s.n, E = s.E, A = (uint64_t)s.T * s.K;
  {
    const uint64_t dims[3] = {n, d, E}, str[2] = {n * 2, d * n * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_map(&f.mg, w_gate, 3, dims, str, box)) return MOE_ERR_CUDA;
    if (!make_map(&f.mu, w_up, 3, dims, str, box)) return MOE_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {n, A}, str[1] = {n * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_map(&f.ma, a_act, 2, dims, str, box)) return MOE_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {d, n, E}, str[2] = {d * 2, n * d * 2};
    const uint32_t box[3] = {64, 64, 1};
    if (!make_map(&f.md, w_down, 3, dims, str, box)) return MOE_ERR_CUDA;
  }
  GemmArgs& ga = f.gate_up;
  ga.offsets = offsets;
  ga.p2a = p2a;
  ga.x = (const uint8_t*)x;
  ga.x_row_bytes = (long long)s.d * 2;
  ga.E = s.E;
  ga.K = s.K;
  ga.T = s.T;
  ga.status = device_status_ptr();
  ga.limit_ns = kWaitLimitNs;
  ga.h_out = nullptr;
  ga.out = (bf16*)a_act;
  ga.ld_out = s.n;
  ga.n_out = s.n;
  ga.out_tile = 128;
  ga.n_tiles = (s.n + 127) / 128;
  ga.kblocks = s.d / BK;
  ga.kb_split = ga.kblocks;
  GemmArgs& gd = f.down;
  gd = ga;
  gd.out = (bf16*)y_perm;
  gd.ld_out = s.d;
  gd.n_out = s.d;
  gd.out_tile = BN;
  gd.n_tiles = (s.d + BN - 1) / BN;
  gd.kblocks = s.n / BK;
  gd.kb_split = gd.kblocks;
  return MOE_OK;
}

moe_status launch_ffn_tc2_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0,
                               const CUtensorMap& b1, const GemmArgs& args, cudaStream_t st);
moe_status launch_gather_rows(const moe_shape& s, const void* x, const int32_t* p2a,
                              const int32_t* offsets, void* x_perm, cudaStream_t st);

// h_out (nullable): the gate/up pre-activations (g | u) of every kept row, for the backward
// (single-CTA tiles then). gateup_mode 0: single-CTA tiles, A rows gathered in the kernel;
// 1: CTA pairs, A rows
// gathered in the kernel; 2: the rows are first copied expert-major into y_perm (which the
// down GEMM overwrites only later), then CTA pairs load A from there by TMA.
moe_status launch_ffn_tc_mixed(const moe_shape& s, const void* x, const int32_t* offsets,
                               const int32_t* p2a, const void* w_gate, const void* w_up,
                               const void* w_down, void* a_act, void* y_perm, int gateup_mode,
                               bool pair_down, void* h_out, cudaStream_t st) {
  if ((long long)s.T * s.K == 0) return MOE_OK;
  FfnMaps f;
  moe_status r = prepare_ffn(s, x, offsets, p2a, w_gate, w_up, w_down, a_act, y_perm, f);
  if (r != MOE_OK) return r;
  f.gate_up.h_out = (bf16*)h_out;
  if (h_out != nullptr) gateup_mode = 0;  // the single-CTA epilogue keeps the pre-activations
  if (gateup_mode == 2) {
    if ((r = launch_gather_rows(s, x, p2a, offsets, y_perm, st)) != MOE_OK) return r;
    CUtensorMap mx;
    const uint64_t dims[2] = {(uint64_t)s.d, (uint64_t)s.T * s.K}, str[1] = {(uint64_t)s.d * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_map(&mx, y_perm, 2, dims, str, box)) return MOE_ERR_CUDA;
    r = launch_ffn_tc2_gemm(2, mx, f.mg, f.mu, f.gate_up, st);
  } else if (gateup_mode == 1) {
    r = launch_ffn_tc2_gemm(1, f.mg, f.mg, f.mu, f.gate_up, st);
  } else {
    r = run_gemm<true>(f.mg, f.mg, f.mu, f.gate_up, st, K_GATEUP_TC);
  }
  if (r != MOE_OK) return r;
  return pair_down ? launch_ffn_tc2_gemm(0, f.ma, f.md, f.md, f.down, st)
                   : run_gemm<false>(f.ma, f.md, f.md, f.down, st, K_DOWN_TC);
}

}  // namespace moe
