// Head-map calibration on sm_100a: the Gram matrix of the stacked sender and receiver maps
// over causal positions (tcgen05 + TMA + TMEM for bf16, SIMT otherwise), and the
// least-squares solve for the head-mapping weights.
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?", section "不传 KV Cache,改传“注意力关系”":
// the weights that combine sender heads into receiver heads are learned once, offline, with
// both models frozen; the page gives no objective.  Reading taken: least squares of every
// receiver head's map Y_r on the sender heads' maps X_s over the causal positions
// (i < L, j <= i), optionally with a ridge term.  Everything the fit needs is the Gram
//   G = sum_pos f f^T,   f = (X_0 .. X_{h_s-1}, Y_0 .. Y_{h_r-1})[i, j],
// a contraction over ~L^2 / 2 positions with F = h_s + h_r <= 128 features: HBM-bound
// (each map byte is read once) but far beyond what SIMT FMAs sustain, so the bf16 path runs
// it on the tensor cores.
//
// Tensor-core kernel.  A tile is one query row i and 64 consecutive keys of it: TMA brings
// the 128-byte rows of all sender heads, then of all receiver heads, into consecutive
// 128-byte rows of shared memory (128-byte swizzle) - a K-major operand whose M (or N)
// index is the feature and whose K index is the key.  D[F][F] += T T^T takes four
// tcgen05.mma (M=128, N=F rounded up to 16, K=16) per tile with A and B both the tile; the
// operand rows past F belong to the next tile or to a zero pad and only reach D rows or
// columns >= F, which are never read.  Keys j > i of the diagonal tile are zeroed in shared
// memory by the MMA warp before the MMAs (keys >= L arrive as zeros: they lie outside the
// tensor map).  Each CTA accumulates a contiguous range of tiles in TMEM (float32) and writes
// its partial Gram; a second kernel adds the partials into the caller's double Gram in a
// fixed order.  Roles: warp 0 TMA producer, warp 1 masking + MMA issue + TMEM owner, warps
// 2-5 read D.  Every wait is bounded; on expiry the CTA records ST_TIMEOUT and stops.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "mf_internal.cuh"

namespace mfi {
namespace {

constexpr int GT = 192;                      // 6 warps
constexpr int KEYS = 64;                     // keys per tile (one 128-byte row per head)
constexpr int G_STAGES = 2;                   // two large stages: each stage costs a fixed
constexpr uint32_t G_STAGE_BYTES = 96 * 1024;  // hand-off (~0.6 us) beside its tiles' share
constexpr uint32_t G_PAD_BYTES = 128 * 128;  // rows an M=128 operand may read past the last tile
constexpr uint32_t G_OFF_BAR = G_STAGES * G_STAGE_BYTES + G_PAD_BYTES;
constexpr uint32_t G_SMEM = G_OFF_BAR + 256 + 1024;  // + alignment slack
constexpr int FMAX_TC = 128, FMAX_SIMT = 64, HMAX = 64;

struct GramParams {
  int L, h_s, h_r, F, F8, Fn;  // F8: shared-memory rows per tile, Fn: MMA N
  int tps;                     // tiles per stage
  int64_t n_tiles;             // sum over rows i < L of (floor(i / 64) + 1)
  double* partial;             // [gridDim.x][F][F]
  uint32_t* status;
  uint64_t wait_ns;            // limit of every pipeline wait
  int stall;                   // test: the MMA warp first waits on a barrier nothing arrives at
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t su32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_init(uint32_t b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_expect(uint32_t b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(b), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait: false (and ST_TIMEOUT, abort flag) after limit_ns or once another role has
// given up
__device__ __forceinline__ bool bar_wait(uint32_t b, uint32_t parity, volatile int* abort_flag,
                                         uint32_t* status, uint64_t limit_ns) {
  if (bar_try(b, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t it = 1;; ++it) {
    if (bar_try(b, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (gtimer() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(status, ST_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma3(uint32_t dst, const CUtensorMap* tm, uint32_t b, int c0,
                                     int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(b), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void commit(uint32_t b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(b)
               : "memory");
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t bdesc, uint32_t idesc,
                                    uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t kmajor_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024u >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                 "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                 "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                 "+r"(v[30]), "+r"(v[31]));
}

// tile t of a sequence -> (query row i, key chunk c): rows 64a .. 64a+63 have a + 1 tiles
// each, and 32 a (a + 1) tiles come before row 64a
__host__ __device__ inline void tile_of(int64_t t, int* i, int* c) {
  int a = (int)((sqrtf(1.0f + (float)t * 0.125f) - 1.0f) * 0.5f);  // corrected below
  while (32ll * (a + 1) * (a + 2) <= t) ++a;
  while (a > 0 && 32ll * a * (a + 1) > t) --a;
  const int64_t rem = t - 32ll * a * (a + 1);
  *i = 64 * a + (int)(rem / (a + 1));
  *c = (int)(rem % (a + 1));
}
// the tile after (i, c) in that order
__host__ __device__ inline void next_tile(int* i, int* c) {
  if (*c < (*i >> 6)) ++*c;
  else { ++*i; *c = 0; }
}
inline int64_t tiles_of_length(int L) {
  const int64_t A = L / 64, rest = L - 64 * A;
  return 32 * A * (A + 1) + rest * (A + 1);
}

// ------------------------------------------------------------------ tcgen05 Gram
__global__ void __launch_bounds__(GT, 1)
    k_calib_gram_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                    GramParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sb = su32(smem);
  const uint32_t bar0 = sb + G_OFF_BAR;
  auto FULL = [&](int s) { return bar0 + 8u * (uint32_t)s; };
  auto EMPTY = [&](int s) { return bar0 + 8u * (uint32_t)(G_STAGES + s); };
  const uint32_t DONE = bar0 + 8u * (2 * G_STAGES);
  const uint32_t NEVER = bar0 + 8u * (2 * G_STAGES + 1);  // test stall: nothing arrives here
  const uint32_t tile_bytes = (uint32_t)p.F8 * 128u;

  // stages of p.tps consecutive tiles, dealt round-robin: global stage g goes to CTA
  // g % gridDim.x, so the CTAs work on neighbouring rows at the same time (the rows of all head
  // planes they touch share pages: far fewer translation misses than one contiguous range per CTA)
  const int64_t n_stages = (p.n_tiles + p.tps - 1) / p.tps;
  const int n_st = blockIdx.x < n_stages ? (int)((n_stages - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  auto stage_tiles = [&](int st, int64_t* ta, int* n) {
    *ta = ((int64_t)blockIdx.x + (int64_t)st * gridDim.x) * p.tps;
    *n = (int)(p.n_tiles - *ta < (int64_t)p.tps ? p.n_tiles - *ta : (int64_t)p.tps);
  };

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < G_STAGES; ++s) {
      bar_init(FULL(s), 1);
      bar_init(EMPTY(s), 1);
    }
    bar_init(DONE, 1);
    bar_init(NEVER, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the pad an M=128 operand may read past the last tile of the last stage
  for (uint32_t k = threadIdx.x; k < G_PAD_BYTES / 16; k += GT)
    reinterpret_cast<uint4*>(smem + G_STAGES * G_STAGE_BYTES)[k] = make_uint4(0, 0, 0, 0);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(&s_tmem)),
                 "r"(128)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ================================================================ TMA producer
    // the whole warp waits (suspended by the hardware, where a lone polling lane would spin);
    // lane 0 issues the copies
    bool ok = true;
    int issued = 0;
    for (int st = 0; st < n_st && ok; ++st) {
      const int s = st % G_STAGES;
      ok = __all_sync(0xffffffffu, bar_wait(EMPTY(s), ((st / G_STAGES) & 1) ^ 1, abort_flag, p.status, p.wait_ns));
      if (!ok) break;
      int64_t ta;
      int n;
      stage_tiles(st, &ta, &n);
      if (lane == 0) {
        bar_expect(FULL(s), (uint32_t)(n * (p.h_s + p.h_r) * 128));
        int i, c;  // the stage's first tile, then stepped along (no square root per tile)
        tile_of(ta, &i, &c);
        for (int k = 0; k < n; ++k, next_tile(&i, &c)) {
          const uint32_t dst = sb + s * G_STAGE_BYTES + k * tile_bytes;
          tma3(dst, &tmX, FULL(s), c * KEYS, 0, i);
          tma3(dst + p.h_s * 128u, &tmY, FULL(s), c * KEYS, 0, i);
        }
      }
      __syncwarp();
      ++issued;
    }
    // drain: wait (bounded) for the last copies issued into every stage
    if (lane == 0)
      for (int s = 0; s < G_STAGES; ++s) {
        const int cnt = issued > s ? (issued - s - 1) / G_STAGES + 1 : 0;
        if (cnt) {
          const uint64_t w0 = gtimer();
          while (!bar_try(FULL(s), (cnt - 1) & 1) && gtimer() - w0 < DRAIN_NS) {}
        }
      }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ mask + MMA issue
    // D[f][g] += sum_k T[f][k] T[g][k]: M=128 (rows past F are ignored), N=Fn, K=16
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.Fn >> 3) << 17) |
                           ((128u >> 4) << 24);
    bool ok = true;
    // test stall: a wait that can only run out (the whole CTA then stops as on any timeout)
    if (p.stall) ok = __all_sync(0xffffffffu, bar_wait(NEVER, 0, abort_flag, p.status, p.wait_ns));
    for (int st = 0; st < n_st && ok; ++st) {
      const int s = st % G_STAGES;
      ok = __all_sync(0xffffffffu, bar_wait(FULL(s), (st / G_STAGES) & 1, abort_flag, p.status, p.wait_ns));
      if (!ok) break;
      int64_t ta;
      int n;
      stage_tiles(st, &ta, &n);
      // keys j > i of a diagonal tile do not count: zero them in every feature row
      int i, c;
      tile_of(ta, &i, &c);
      for (int k = 0; k < n; ++k, next_tile(&i, &c)) {
        const int r0 = i & 63;
        if (c != (i >> 6) || r0 == 63) continue;
        uint8_t* tb = smem + s * G_STAGE_BYTES + k * tile_bytes;
        for (int e = lane; e < p.F * 8; e += 32) {
          const int row = e >> 3, q = e & 7;  // 16-byte chunk q holds keys 8q .. 8q+7
          if (8 * q + 7 <= r0) continue;
          uint8_t* chunk = tb + row * 128 + ((q ^ (row & 7)) << 4);
          if (8 * q > r0) {
            *reinterpret_cast<uint4*>(chunk) = make_uint4(0, 0, 0, 0);
          } else {
            for (int x = r0 - 8 * q + 1; x < 8; ++x) reinterpret_cast<uint16_t*>(chunk)[x] = 0;
          }
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        fence_after();
        for (int k = 0; k < n; ++k) {
          const uint64_t dsc = kmajor_sw128(sb + s * G_STAGE_BYTES + k * tile_bytes);
#pragma unroll
          for (int kk = 0; kk < KEYS / 16; ++kk)  // +32 bytes per 16 keys
            mma(tmem, dsc + 2u * kk, dsc + 2u * kk, idesc, (st > 0 || k > 0 || kk > 0) ? 1u : 0u);
        }
        commit(EMPTY(s));
      }
      __syncwarp();
    }
    if (lane == 0) {
      commit(DONE);
      const uint64_t w0 = gtimer();
      while (!bar_try(DONE, 0) && gtimer() - w0 < DRAIN_NS) {}
    }
    __syncwarp();
  } else {
    // ================================================================ read D
    bool ok = __all_sync(0xffffffffu, bar_wait(DONE, 0, abort_flag, p.status, p.wait_ns));
    if (ok) {
      fence_after();
      const int q = warp & 3;  // TMEM lane quarter of this warp
      const int row = q * 32 + lane;
      double* out = p.partial + (int64_t)blockIdx.x * p.F * p.F;
      for (int c0 = 0; c0 < p.Fn; c0 += 32) {
        uint32_t v[32];
        ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
        if (row < p.F)
#pragma unroll
          for (int cc = 0; cc < 32; ++cc)
            if (c0 + cc < p.F) out[(int64_t)row * p.F + c0 + cc] = (double)__uint_as_float(v[cc]);
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128)
                 : "memory");
  }
}

// ------------------------------------------------------------------ SIMT Gram
template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// One block per stretch of tiles; the tile's features [F][64] are staged in shared memory
// (keys j > i and j >= L as zeros) and every thread accumulates its (f, g) pairs in double.
template <typename T>
__global__ void __launch_bounds__(256) k_calib_gram_simt(const T* X, const T* Y, int64_t Lp,
                                                         GramParams p) {
  __shared__ float tile[FMAX_SIMT][KEYS];
  const int F = p.F, pairs = F * F;
  double acc[FMAX_SIMT * FMAX_SIMT / 256];
#pragma unroll
  for (int k = 0; k < FMAX_SIMT * FMAX_SIMT / 256; ++k) acc[k] = 0.0;
  const int64_t t0 = p.n_tiles * blockIdx.x / gridDim.x, t1 = p.n_tiles * (blockIdx.x + 1) / gridDim.x;
  for (int64_t t = t0; t < t1; ++t) {
    int i, c;
    tile_of(t, &i, &c);
    __syncthreads();
    for (int e = threadIdx.x; e < F * KEYS; e += 256) {
      const int f = e / KEYS, jj = e % KEYS, j = c * KEYS + jj;
      float v = 0.0f;
      if (j <= i && j < p.L)
        v = f < p.h_s ? to_f(X[((int64_t)f * Lp + i) * Lp + j])
                      : to_f(Y[((int64_t)(f - p.h_s) * Lp + i) * Lp + j]);
      tile[f][jj] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < FMAX_SIMT * FMAX_SIMT / 256; ++k) {
      const int e = threadIdx.x + 256 * k;
      if (e < pairs) {
        const int f = e / F, g = e % F;
        float s = 0.0f;  // 64 products in float, tiles added in double
        for (int jj = 0; jj < KEYS; ++jj) s = fmaf(tile[f][jj], tile[g][jj], s);
        acc[k] += (double)s;
      }
    }
  }
  double* out = p.partial + (int64_t)blockIdx.x * pairs;
#pragma unroll
  for (int k = 0; k < FMAX_SIMT * FMAX_SIMT / 256; ++k) {
    const int e = threadIdx.x + 256 * k;
    if (e < pairs) out[e] = acc[k];
  }
}

// gram += sum of the partials, in block order (the same sum on every run)
__global__ void k_calib_reduce(const double* partial, int nparts, int pairs, double* gram) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= pairs) return;
  double s = 0.0;
  for (int b = 0; b < nparts; ++b) s += partial[(int64_t)b * pairs + e];
  gram[e] += s;
}

// Cholesky of G_ss + ridge I (column by column: thread 0 takes the pivot, threads t > c the
// column below it), then each warp solves the two triangular systems of one receiver head at a
// time (lanes over the sender heads, warp-shuffle sums) and forms its residual sum of squares.
// Working storage is static shared memory only.  Square roots and divisions go through the
// reciprocal square root of each pivot, refined in double by Newton-Raphson
// (y <- y (3 - d y^2) / 2, quadratic convergence from a float32 start), so the factor holds
// 1 / L_cc and every division becomes a multiplication.
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double rsqrt_newton(double d) {
  double y = (double)rsqrtf((float)d);  // ~23 bits
#pragma unroll
  for (int it = 0; it < 3; ++it) y = y * (1.5 - 0.5 * d * y * y);
  return y;
}

__global__ void __launch_bounds__(HMAX) k_calib_solve(const double* gram, int h_s, int h_r,
                                                      double ridge, float* W, double* residual,
                                                      uint32_t* status) {
  __shared__ double Lf[HMAX][HMAX];
  __shared__ double inv_diag[HMAX];        // 1 / L_cc
  __shared__ double vec[HMAX / 32][HMAX];  // per warp: forward, then (in place) backward solution
  __shared__ int bad;
  const int t = threadIdx.x, lane = t & 31, wp = t >> 5;
  if (h_s < 1 || h_s > HMAX || h_r < 1 || h_r > HMAX || blockDim.x != HMAX) {
    if (t == 0) atomicOr(status, ST_INDEX);
    return;
  }
  const int F = h_s + h_r;
  if (t == 0) bad = 0;
  __syncthreads();
  for (int c = 0; c < h_s; ++c) {
    if (t == 0) {
      double d = gram[c * F + c] + ridge;
      for (int k = 0; k < c; ++k) d -= Lf[c][k] * Lf[c][k];
      if (!(d > 0.0) || !(d < 1e300)) {
        bad = 1;
      } else {
        const double y = rsqrt_newton(d);
        Lf[c][c] = d * y;
        inv_diag[c] = y;
      }
    }
    __syncthreads();
    if (bad) break;
    if (t > c && t < h_s) {
      double v = gram[t * F + c];
      for (int k = 0; k < c; ++k) v -= Lf[t][k] * Lf[c][k];
      Lf[t][c] = v * inv_diag[c];
    }
    __syncthreads();
  }
  if (bad) {
    if (t == 0) atomicOr(status, ST_SINGULAR);
    for (int e = t; e < h_r * h_s; e += blockDim.x) W[e] = 0.0f;
    if (residual && t < h_r) residual[t] = 0.0;
    return;
  }
  double* w = vec[wp];
  for (int r = wp; r < h_r; r += HMAX / 32) {
    for (int a = 0; a < h_s; ++a) {  // L z = c_r
      double part = 0.0;
      for (int k = lane; k < a; k += 32) part += Lf[a][k] * w[k];
      const double dot = warp_sum(part);
      if (lane == 0) w[a] = (gram[a * F + h_s + r] - dot) * inv_diag[a];
      __syncwarp();
    }
    for (int a = h_s - 1; a >= 0; --a) {  // L^T w = z, in place
      double part = 0.0;
      for (int k = a + 1 + lane; k < h_s; k += 32) part += Lf[k][a] * w[k];
      const double dot = warp_sum(part);
      if (lane == 0) w[a] = (w[a] - dot) * inv_diag[a];
      __syncwarp();
    }
    double part = 0.0;  // residual: Syy - 2 w.c + w^T G w
    for (int a = lane; a < h_s; a += 32) {
      double gw = 0.0;
      for (int b = 0; b < h_s; ++b) gw += gram[a * F + b] * w[b];
      part += w[a] * (gw - 2.0 * gram[a * F + h_s + r]);
      W[r * h_s + a] = (float)w[a];
    }
    const double res = gram[(h_s + r) * F + h_s + r] + warp_sum(part);
    if (residual && lane == 0) residual[r] = res;
    __syncwarp();
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// one sequence's maps [h][Lp][Lp] bf16 as (key j < L, head, row i < L), box (64, h, 1)
bool encode_maps(CUtensorMap* tm, const void* base, int h, int L, int64_t Lp, std::string* err) {
  auto fn = encode_fn();
  if (!fn) { *err = "cuTensorMapEncodeTiled unavailable"; return false; }
  const cuuint64_t dims[3] = {(cuuint64_t)L, (cuuint64_t)h, (cuuint64_t)L};
  const cuuint64_t strides[2] = {(cuuint64_t)(Lp * Lp * 2), (cuuint64_t)(Lp * 2)};
  const cuuint32_t box[3] = {KEYS, (cuuint32_t)h, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { *err = "cuTensorMapEncodeTiled failed: " + std::to_string((int)r); return false; }
  return true;
}

int sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace

int calib_path(const mf_calib_desc& d) {
  const int F = d.h_s + d.h_r;
  return (d.dtype == MF_BF16 && d.h_s % 8 == 0 && F <= FMAX_TC) ? 1 : 0;
}

size_t calib_ws_bytes(const mf_calib_desc& d) {
  const int F = d.h_s + d.h_r;
  // partial Grams of at most 2 x SMs blocks (SIMT) or SMs CTAs (tcgen05)
  return (size_t)2 * sms() * F * F * sizeof(double);
}

bool launch_calib_gram(const mf_calib_desc& d, void* ws, uint32_t* status, cudaStream_t st,
                       std::string* err) {
  const int F = d.h_s + d.h_r;
  const bool tc = calib_path(d) == 1;
  if (!tc && F > FMAX_SIMT) { *err = "h_s + h_r > 64 needs bf16 maps with h_s % 8 == 0"; return false; }
  const size_t esz = d.dtype == MF_BF16 ? 2 : 4;
  for (int s = 0; s < d.nseq; ++s) {
    const int L = d.seqlens[s];
    if (L <= 0) continue;
    const int64_t Lp = ((int64_t)L + d.B - 1) / d.B * d.B;
    GramParams p{};
    p.L = L; p.h_s = d.h_s; p.h_r = d.h_r; p.F = F;
    p.F8 = (F + 7) / 8 * 8;
    p.Fn = (F + 15) / 16 * 16;
    p.n_tiles = tiles_of_length(L);
    p.partial = static_cast<double*>(ws);
    p.status = status;
    p.wait_ns = wait_limit_ns();
    p.stall = wait_stall();
    const char* X = static_cast<const char*>(d.sender_maps) + d.sender_seq_offset[s] * esz;
    const char* Y = static_cast<const char*>(d.receiver_maps) + d.receiver_seq_offset[s] * esz;
    int grid;
    if (tc) {
      p.tps = (int)(G_STAGE_BYTES / ((uint32_t)p.F8 * 128u));
      grid = (int)std::min<int64_t>(sms(), (p.n_tiles + p.tps - 1) / p.tps);
      CUtensorMap tmX, tmY;
      if (!encode_maps(&tmX, X, d.h_s, L, Lp, err) || !encode_maps(&tmY, Y, d.h_r, L, Lp, err))
        return false;
      static std::once_flag attr;
      std::call_once(attr, [] {
        cudaFuncSetAttribute(k_calib_gram_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
      });
      k_calib_gram_tc<<<grid, GT, G_SMEM, st>>>(tmX, tmY, p);
    } else {
      grid = (int)std::min<int64_t>(2 * sms(), p.n_tiles);
      if (d.dtype == MF_BF16)
        k_calib_gram_simt<__nv_bfloat16><<<grid, 256, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(X), reinterpret_cast<const __nv_bfloat16*>(Y), Lp, p);
      else
        k_calib_gram_simt<float><<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(X),
                                                        reinterpret_cast<const float*>(Y), Lp, p);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) { *err = std::string("calib gram launch: ") + cudaGetErrorString(e); return false; }
    k_calib_reduce<<<(F * F + 255) / 256, 256, 0, st>>>(p.partial, grid, F * F, d.gram);
    e = cudaGetLastError();
    if (e != cudaSuccess) { *err = std::string("calib reduce launch: ") + cudaGetErrorString(e); return false; }
  }
  return true;
}

cudaError_t launch_calib_solve(const double* gram, int h_s, int h_r, double ridge, float* W,
                               double* residual, uint32_t* status, cudaStream_t st) {
  k_calib_solve<<<1, HMAX, 0, st>>>(gram, h_s, h_r, ridge, W, residual, status);
  return cudaGetLastError();
}

}  // namespace mfi
