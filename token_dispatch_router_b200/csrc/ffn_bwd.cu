// Backward of the expert half of the layer on the tensor cores, without caching Y.
//
// SonicMoE explainer (gitcode.csdn.net), section 6.4: instead of keeping the down-projection
// output Y (and dY), the routing-weight gradient is taken as dS = <dA', A> with
// dA' = dO W_down^T, because out = sum_k w_k Y_k and Y = A W_down give
// dL/dw = <dO, Y> = <dO W_down^T, A>; section 6.2: the rows of dO are gathered by routing
// index inside the GEMM's operand load; section 6.3: the elementwise backward of SwiGLU
// runs in the epilogue while the accumulator is on chip.
//
// One persistent kernel (grid = #SMs, 320 threads, one CTA per SM) computes, for every
// kept slot p of expert e holding token t's slot k (a = perm_to_assign[p]):
//   dA'[p, :] = dO[t, :] W_down[e]^T            (tcgen05, M=128 rows, N=256 of n, K = d)
//   A = silu(g) u, dS[p] = sum_j dA'[p, j] A[p, j], dA = w[t, k] dA'
//   dG = dA u s (1 + g (1 - s)), dU = dA silu(g), s = 1 / (1 + e^-g)
// with g, u read from the pre-activations h[p] = (g | u) that the forward saved.
//   warp 0     TMA producer: the B tile, 256 rows of W_down[e] (n) x 64 of d, one
//              K-major box (128-byte swizzle), into a 4-stage ring (48 KB a stage);
//   warps 6-9  the gathered A tile: 128 rows of dO (row = perm_to_assign[p] / K) x 64 of
//              d by cp.async into the swizzled K-major layout (MODE 0); or (MODE 2) the dO
//              rows are first copied expert-major into a scratch buffer and the producer
//              loads the A tile from there by TMA, which leaves the load/store units to the
//              epilogue;
//   warp 1     TMEM allocation and the MMA thread (both operands K-major);
//   warps 2-5  epilogue: one TMEM lane = one slot per thread; dG and dU (bf16) into
//              d_h[p] = (dG | dU), and this tile's 256-column part of dS into
//              partial[p][n-tile] (fp32).
// A second kernel adds each slot's parts in n-tile order (deterministic) and writes the
// routing-weight gradient d_w[t, k] (0 at dropped slots). Every mbarrier wait is bounded.
#include <string.h>

#include "ffn_args.cuh"
#include "tc_ptx.cuh"

namespace moe {

namespace {

using namespace ptx;

constexpr int BM = 128, BK = 64, BN = 256, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB: 128 dO rows x 64 of d
constexpr int B_BYTES = BN * BK * 2;  // 32 KB: 256 W_down rows (n) x 64 of d
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS_DACT = 320;  // producer, MMA, 4 epilogue warps, 4 gather warps
constexpr int THREADS_DX = 192;    // producer, MMA, 4 epilogue warps
constexpr int GATHER_WARP0 = 6;
constexpr int GATHER_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAXE = 256;
constexpr int SMEM_TAIL = 4096;
// dA' epilogue: per epilogue warp, one 32-row x 32-column chunk of g and of u (then of dG
// and dU), rows padded to 80 bytes so that a thread reading its own row hits distinct banks
constexpr int EPI_ROW = 80;
constexpr int EPI_WARP_BYTES = 2 * 32 * EPI_ROW;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + SMEM_TAIL + 4 * EPI_WARP_BYTES;
// kind::f16: D fp32 (bit 4), A and B bf16 (bits 7-9, 10-12), both K-major (bits 15, 16 = 0),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28
constexpr uint32_t IDESC =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct BwdArgs {
  const int32_t* offsets;    // [E + 1]
  const int32_t* p2a;        // slot -> flat assignment
  const uint8_t* d_out;      // dA': [T, d] rows gathered by token
  long long row_bytes;       // d * 2
  const float* topk_w;       // [T * K]
  const bf16* h;             // [rows, 2n]: g | u per kept slot
  bf16* d_h;                 // dA': [rows, 2n] out (dG | dU); dX: unused
  float* partial;            // dA': [rows, n_tiles]
  bf16* dx_perm;             // dX: [rows, d] out
  int n;                     // dA': output columns (n); dX: output columns (d)
  int n_tiles, kblocks, kb_split, E, K, T;  // dX: k-blocks < kb_split read W_gate, then W_up
  unsigned* status;
  unsigned long long limit_ns;
};

struct Tile {
  int e, m0, rows, n0, nt;
};

__device__ __forceinline__ Tile decode(int w, const int* s_off, const int* s_cum, const int* s_mt,
                                       int E) {
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
  t.nt = local / mt;
  t.n0 = t.nt * BN;
  t.m0 = s_off[lo] + (local % mt) * BM;
  t.rows = min(BM, s_off[lo + 1] - t.m0);
  return t;
}

// MODE 0 (dA'): A = rows of dO gathered by token, B = W_down[e] (K = d), epilogue above.
// MODE 1 (dX): A = the (dG | dU) rows by TMA, B = W_gate[e] for the first n of K and W_up[e]
// for the second (K = 2n), both read K-major in place; epilogue: bf16 dX_perm rows.
// MODE 2 (dA'): as MODE 0 with A = the dO rows copied expert-major beforehand, by TMA.
template <int MODE>
__global__ void __launch_bounds__(MODE == 0 ? THREADS_DACT : THREADS_DX, 1)
    grouped_gemm_bwd(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const BwdArgs g) {
  constexpr int THREADS = MODE == 0 ? THREADS_DACT : THREADS_DX;
  constexpr bool GATHER = MODE == 0;
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
  uint8_t* epi = base + STAGES * STAGE_BYTES + SMEM_TAIL;  // dA' epilogue buffers (16-byte aligned)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = g.E;
  // TMA expect_tx (+ the gather threads' cp.async arrivals in MODE 0)
  constexpr uint32_t FULL_COUNT = GATHER ? 1 + GATHER_THREADS : 1;
  constexpr uint32_t TMA_BYTES = GATHER ? B_BYTES : STAGE_BYTES;

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
    mbar_init_fence();
  }
  if (tid == 32) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    if (!GATHER)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    if (MODE == 1)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB2)) : "memory");
  }
  if (warp == 1) tmem_alloc<1>(saddr(tmem_slot), TMEM_COLS);
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  for (int i = tid; i <= E; i += THREADS) s_off[i] = g.offsets[i];
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
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
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
    // ------------------------------------------------------------ TMA producer (B)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_par = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Tile t = decode(w, s_off, s_cum, s_mt, E);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0)
          w_ok = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, limit);
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t fb = saddr(&full[stage]);
          const uint32_t a_dst = saddr(ring + stage * STAGE_BYTES);
          mbar_expect_tx(fb, TMA_BYTES);
          if (GATHER) {
            tma_load_3d(a_dst + A_BYTES, &tmB, kb * BK, t.n0, t.e, fb);
          } else if (MODE == 2) {
            tma_load_2d(a_dst, &tmA, kb * BK, t.m0, fb);
            tma_load_3d(a_dst + A_BYTES, &tmB, kb * BK, t.n0, t.e, fb);
          } else {
            tma_load_2d(a_dst, &tmA, kb * BK, t.m0, fb);
            if (kb < g.kb_split)
              tma_load_3d(a_dst + A_BYTES, &tmB, kb * BK, t.n0, t.e, fb);
            else
              tma_load_3d(a_dst + A_BYTES, &tmB2, (kb - g.kb_split) * BK, t.n0, t.e, fb);
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
    if (lane == 0) {  // drain: the last load issued into each stage has landed (bounded)
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
        if (!mbar_wait(saddr(&tempty[buf]), (use & 1u) ^ 1u, abort_flag, g.status, limit)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(saddr(&full[stage]), phase, abort_flag, g.status, limit)) {
            ok = false;
            break;
          }
          if (GATHER) fence_proxy_async_smem();  // cp.async (generic) writes -> MMA reads
          tc_fence_after();
          const uint32_t a_addr = saddr(ring + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = desc_sw128(b_addr + kk * 32, 16, 1024);
            tc_mma<1>(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit<1>(saddr(&empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) tc_commit<1>(saddr(&tfull[buf]));
      }
      tc_commit<1>(saddr(done));  // every MMA completed before TMEM is released (bounded)
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try(saddr(done), 0) && globaltimer_ns() - t0 < limit) {
      }
    }
  } else if (GATHER && warp >= GATHER_WARP0) {
    // ------------------------------------------------------------ A gather: rows of dO
    const int gw = warp - GATHER_WARP0;
    const int c = lane & 7;
    const int rg = lane >> 3;
    int stage = 0;
    uint32_t phase = 0;
    auto rows_of = [&](int w, const uint8_t* (&src)[8]) {
      const Tile t = decode(w, s_off, s_cum, s_mt, E);
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
        src[i] = g.d_out + (size_t)tk * g.row_bytes + c * 16;
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
      const uint8_t* nsrc[8];
      if (w + (int)gridDim.x < total) rows_of(w + gridDim.x, nsrc);
      bool ok = true;
      for (int kb = 0; kb < g.kblocks; ++kb) {
        int w_ok = 0;
        if (lane == 0)
          w_ok = mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, g.status, limit);
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
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const size_t ld = 2 * (size_t)g.n;  // h and d_h row length
    int it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      const Tile t = decode(w, s_off, s_cum, s_mt, E);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      int w_ok = 0;
      if (lane == 0) w_ok = mbar_wait(saddr(&tfull[buf]), use & 1u, abort_flag, g.status, limit);
      w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
      if (!w_ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (uint32_t)(buf * BN) + ((uint32_t)(q * 32) << 16);
      const bool row_ok = r < t.rows;
      const int p = t.m0 + (row_ok ? r : 0);
      if (MODE == 1) {  // dX_perm rows, bf16
        bf16* orow = g.dx_perm + (size_t)p * g.n;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tb + c * 32, v);
          tmem_ld_wait();
          const int col = t.n0 + c * 32;
          if (row_ok && col < g.n) {
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
        tc_fence_before();
        mbar_arrive(saddr(&tempty[buf]));
        continue;
      }
      const float wt = row_ok ? g.topk_w[g.p2a[p]] : 0.f;
      float ds = 0.f;
      // The warp's 32 rows of a 32-column chunk of g and u are loaded cooperatively (a lane
      // moves 16 of a row's 64 bytes; one instruction covers 8 whole row segments), put
      // through the warp's padded buffer so that each thread reads its own row, and dG / dU
      // go back out the same way. The next chunk's loads are issued before this chunk's math.
      uint8_t* gbuf = epi + q * EPI_WARP_BYTES;
      uint8_t* ubuf = gbuf + 32 * EPI_ROW;
      const int lr = lane >> 2, lc = lane & 3;  // this lane's row (of 8) and 16-byte column
      uint4 gn[4], un[4];
      auto load_chunk = [&](int c) {
        const int col = t.n0 + c * 32 + lc * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int rr = q * 32 + lr + 8 * i;  // row inside the tile
          if (rr < t.rows && col < g.n) {
            const bf16* src = g.h + (size_t)(t.m0 + rr) * ld + col;
            gn[i] = *reinterpret_cast<const uint4*>(src);
            un[i] = *reinterpret_cast<const uint4*>(src + g.n);
          } else {
            gn[i] = make_uint4(0, 0, 0, 0);
            un[i] = gn[i];
          }
        }
      };
      load_chunk(0);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          *reinterpret_cast<uint4*>(gbuf + (lr + 8 * i) * EPI_ROW + lc * 16) = gn[i];
          *reinterpret_cast<uint4*>(ubuf + (lr + 8 * i) * EPI_ROW + lc * 16) = un[i];
        }
        __syncwarp();
        uint4 gq[4], uq[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          gq[j] = *reinterpret_cast<const uint4*>(gbuf + lane * EPI_ROW + j * 16);
          uq[j] = *reinterpret_cast<const uint4*>(ubuf + lane * EPI_ROW + j * 16);
        }
        uint32_t v[32];
        tmem_ld32(tb + c * 32, v);
        if (c + 1 < BN / 32) load_chunk(c + 1);
        tmem_ld_wait();
        const int col = t.n0 + c * 32;
        uint32_t pg[16], pu[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float gf[8], uf[8];
          unpack16(gq[j], gf, bf16());
          unpack16(uq[j], uf, bf16());
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            float dg[2], du[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const float gg = gf[i + h2], uu = uf[i + h2];
              const float da1 = __uint_as_float(v[8 * j + i + h2]);
              const float s = __fdividef(1.f, 1.f + __expf(-gg));
              const float silu = gg * s;
              if (row_ok) ds = fmaf(da1, silu * uu, ds);
              const float da = wt * da1;
              dg[h2] = da * uu * s * (1.f + gg * (1.f - s));
              du[h2] = da * silu;
            }
            pg[4 * j + i / 2] = pack_bf16x2(dg[0], dg[1]);
            pu[4 * j + i / 2] = pack_bf16x2(du[0], du[1]);
          }
        }
        __syncwarp();  // every lane has read its g and u rows
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          *reinterpret_cast<uint4*>(gbuf + lane * EPI_ROW + j * 16) =
              make_uint4(pg[4 * j], pg[4 * j + 1], pg[4 * j + 2], pg[4 * j + 3]);
          *reinterpret_cast<uint4*>(ubuf + lane * EPI_ROW + j * 16) =
              make_uint4(pu[4 * j], pu[4 * j + 1], pu[4 * j + 2], pu[4 * j + 3]);
        }
        __syncwarp();
        if (col < g.n) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int rr = q * 32 + lr + 8 * i;
            if (rr < t.rows) {
              bf16* dst = g.d_h + (size_t)(t.m0 + rr) * ld + col + lc * 8;
              *reinterpret_cast<uint4*>(dst) =
                  *reinterpret_cast<const uint4*>(gbuf + (lr + 8 * i) * EPI_ROW + lc * 16);
              *reinterpret_cast<uint4*>(dst + g.n) =
                  *reinterpret_cast<const uint4*>(ubuf + (lr + 8 * i) * EPI_ROW + lc * 16);
            }
          }
        }
        __syncwarp();  // the buffer is free for the next chunk
      }
      if (row_ok) g.partial[(size_t)p * g.n_tiles + t.nt] = ds;
      tc_fence_before();
      mbar_arrive(saddr(&tempty[buf]));
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, TMEM_COLS);
  }
}

// d_w[a] = sum over the n-tiles of slot assign_to_perm[a], in n-tile order; 0 if dropped.
__global__ void __launch_bounds__(256) dw_kernel(const int32_t* __restrict__ a2p,
                                                 const float* __restrict__ partial, int n_tiles,
                                                 long long A, float* __restrict__ d_w) {
  pdl_wait();  // the previous kernel in the stream has completed
  pdl_trigger();
  for (long long a = (long long)blockIdx.x * blockDim.x + threadIdx.x; a < A;
       a += (long long)gridDim.x * blockDim.x) {
    const int p = a2p[a];
    float s = 0.f;
    if (p >= 0)
      for (int j = 0; j < n_tiles; ++j) s += partial[(size_t)p * n_tiles + j];
    d_w[a] = s;
  }
}

}  // namespace

namespace {
size_t align256b(size_t v) { return (v + 255) & ~(size_t)255; }
}  // namespace

// Scratch: the per-slot partial sums of dS, then (when the input gradient is wanted) the
// dX_perm rows.
// The dO rows are copied expert-major before the dA' GEMM (ffn_variant 3), or gathered
// inside it (1, 2). Automatic (0): copied when n >= 4096. The in-GEMM gather shares the
// load/store units with this epilogue's h reads and d_h writes; at n = 14336 the TMA-fed
// GEMM measured 0.870 ms against 0.950 ms, while the copy costs 4 T K d bytes of traffic
// (about 15 us there), a share of the GEMM that grows as n shrinks.
bool backward_copies_rows(const moe_shape& s) {
  return s.ffn_variant == 3 || (s.ffn_variant == 0 && s.n >= 4096);
}

// Scratch: the per-slot partial sums of d_w, then (at backward_rows_offset) one
// [T*K, d] bf16 row buffer: the copied dO rows for the dA' GEMM, later the dX_perm rows.
size_t backward_rows_offset(const moe_shape& s) {
  const size_t n_tiles = (size_t)(s.n + BN - 1) / BN;
  return align256b((size_t)s.T * s.K * n_tiles * sizeof(float));
}

size_t backward_scratch_bytes(const moe_shape& s, bool with_dx) {
  size_t b = backward_rows_offset(s);
  if (with_dx || backward_copies_rows(s)) b += align256b((size_t)s.T * s.K * s.d * 2);
  return b;
}

moe_status launch_combine(const moe_shape& s, const void* y_perm, const int32_t* a2p,
                          const float* topk_w, void* out, cudaStream_t st);
moe_status launch_ffn_tc2_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0,
                               const CUtensorMap& b1, const GemmArgs& args, cudaStream_t st);

// dX on CTA pairs (256-row tiles) when a pair variant is asked for (ffn_variant 2 or 3),
// else on single CTAs: at the Mixtral-like shape the pairs measured slower (1.75-1.79
// against 1.64-1.67 ms), their 256-row tiles padding twice the rows of the 128-row ones.
bool backward_pair_dx(const moe_shape& s) { return s.ffn_variant >= 2; }
moe_status launch_gather_rows(const moe_shape& s, const void* x, const int32_t* p2a,
                              const int32_t* offsets, void* x_perm, cudaStream_t st);

moe_status launch_backward(const moe_shape& s, const void* d_out, const float* topk_w,
                           const int32_t* offsets, const int32_t* p2a, const int32_t* a2p,
                           const void* w_gate, const void* w_up, const void* w_down,
                           const void* h, void* d_h, float* d_w, void* d_x, void* scratch,
                           cudaStream_t st) {
  const long long A = (long long)s.T * s.K;
  if (A == 0) return MOE_OK;
  CUtensorMap mb, none;
  memset(&none, 0, sizeof(none));
  {
    const uint64_t dims[3] = {(uint64_t)s.d, (uint64_t)s.n, (uint64_t)s.E};
    const uint64_t str[2] = {(uint64_t)s.d * 2, (uint64_t)s.n * s.d * 2};
    const uint32_t box[3] = {BK, BN, 1};
    if (!make_map(&mb, w_down, 3, dims, str, box)) return MOE_ERR_CUDA;
  }
  BwdArgs a;
  a.offsets = offsets;
  a.p2a = p2a;
  a.d_out = (const uint8_t*)d_out;
  a.row_bytes = (long long)s.d * 2;
  a.topk_w = topk_w;
  a.h = (const bf16*)h;
  a.d_h = (bf16*)d_h;
  a.partial = (float*)scratch;
  a.dx_perm = nullptr;
  a.n = s.n;
  a.n_tiles = (s.n + BN - 1) / BN;
  a.kblocks = s.d / BK;
  a.kb_split = a.kblocks;
  a.E = s.E;
  a.K = s.K;
  a.T = s.T;
  a.status = device_status_ptr();
  a.limit_ns = kWaitLimitNs;
  bf16* rows = (bf16*)((uint8_t*)scratch + backward_rows_offset(s));
  moe_status r;
  if (backward_copies_rows(s)) {  // dO rows expert-major, then the GEMM loads them by TMA
    if ((r = launch_gather_rows(s, d_out, p2a, offsets, rows, st)) != MOE_OK) return r;
    CUtensorMap ma;
    const uint64_t dims[2] = {(uint64_t)s.d, (uint64_t)A};
    const uint64_t str[1] = {(uint64_t)s.d * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_map(&ma, rows, 2, dims, str, box)) return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(grouped_gemm_bwd<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_begin(K_BWD_ACT, st);
    launch_kernel(grouped_gemm_bwd<2>, dim3((unsigned)sm_count()), dim3(THREADS_DX),
                  (size_t)SMEM_BYTES, st, 1, ma, mb, none, a);
  } else {
    if (cudaFuncSetAttribute(grouped_gemm_bwd<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_begin(K_BWD_ACT, st);
    launch_kernel(grouped_gemm_bwd<0>, dim3((unsigned)sm_count()), dim3(THREADS_DACT),
                  (size_t)SMEM_BYTES, st, 1, none, mb, none, a);
  }
  if ((r = launch_end(K_BWD_ACT, st)) != MOE_OK) return r;
  long long blocks = (A + 255) / 256;
  if (blocks > (long long)sm_count() * 8) blocks = (long long)sm_count() * 8;
  launch_begin(K_BWD_DW, st);
  launch_kernel(dw_kernel, dim3((unsigned)blocks), dim3(256), 0, st, 1, a2p,
                (const float*)scratch, a.n_tiles, A, d_w);
  if ((r = launch_end(K_BWD_DW, st)) != MOE_OK) return r;
  if (d_x == nullptr) return MOE_OK;
  // input gradient: dX_perm = (dG | dU) [W_gate | W_up]^T per expert, then the scatter-add
  bf16* dx_perm = rows;
  if (backward_pair_dx(s)) {
    CUtensorMap pa, pg, pu;
    {
      const uint64_t dims[2] = {2 * (uint64_t)s.n, (uint64_t)A};
      const uint64_t str[1] = {2 * (uint64_t)s.n * 2};
      const uint32_t box[2] = {BK, 128};
      if (!make_map(&pa, d_h, 2, dims, str, box)) return MOE_ERR_CUDA;
    }
    {
      const uint64_t dims[3] = {(uint64_t)s.n, (uint64_t)s.d, (uint64_t)s.E};
      const uint64_t str[2] = {(uint64_t)s.n * 2, (uint64_t)s.d * s.n * 2};
      const uint32_t box[3] = {BK, 128, 1};  // this CTA's 128 of the pair's 256 output columns
      if (!make_map(&pg, w_gate, 3, dims, str, box)) return MOE_ERR_CUDA;
      if (!make_map(&pu, w_up, 3, dims, str, box)) return MOE_ERR_CUDA;
    }
    GemmArgs ga = {};
    ga.offsets = offsets;
    ga.p2a = p2a;
    ga.out = dx_perm;
    ga.ld_out = s.d;
    ga.n_out = s.d;
    ga.out_tile = 256;
    ga.n_tiles = (s.d + 255) / 256;
    ga.kblocks = 2 * s.n / BK;
    ga.kb_split = s.n / BK;
    ga.E = s.E;
    ga.K = s.K;
    ga.T = s.T;
    ga.status = device_status_ptr();
    ga.limit_ns = kWaitLimitNs;
    if ((r = launch_ffn_tc2_gemm(3, pa, pg, pu, ga, st)) != MOE_OK) return r;
    return launch_combine(s, dx_perm, a2p, nullptr, d_x, st);  // unit weights: a plain sum
  }
  CUtensorMap ma, mg, mu;
  {
    const uint64_t dims[2] = {2 * (uint64_t)s.n, (uint64_t)A};
    const uint64_t str[1] = {2 * (uint64_t)s.n * 2};
    const uint32_t box[2] = {BK, BM};
    if (!make_map(&ma, d_h, 2, dims, str, box)) return MOE_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {(uint64_t)s.n, (uint64_t)s.d, (uint64_t)s.E};
    const uint64_t str[2] = {(uint64_t)s.n * 2, (uint64_t)s.d * s.n * 2};
    const uint32_t box[3] = {BK, BN, 1};
    if (!make_map(&mg, w_gate, 3, dims, str, box)) return MOE_ERR_CUDA;
    if (!make_map(&mu, w_up, 3, dims, str, box)) return MOE_ERR_CUDA;
  }
  BwdArgs b = a;
  b.dx_perm = dx_perm;
  b.n = s.d;
  b.n_tiles = (s.d + BN - 1) / BN;
  b.kblocks = 2 * s.n / BK;
  b.kb_split = s.n / BK;
  if (cudaFuncSetAttribute(grouped_gemm_bwd<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  launch_begin(K_BWD_DX, st);
  launch_kernel(grouped_gemm_bwd<1>, dim3((unsigned)sm_count()), dim3(THREADS_DX),
                (size_t)SMEM_BYTES, st, 1, ma, mg, mu, b);
  if ((r = launch_end(K_BWD_DX, st)) != MOE_OK) return r;
  return launch_combine(s, dx_perm, a2p, nullptr, d_x, st);  // unit weights: a plain sum
}

}  // namespace moe
