// Compression straight from the sender's queries and keys on sm_100a: no dense map exists at
// any point.
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com), section
// "存不下、读得慢?三个工程优化手段", subsection 1 "只存重要的:块稀疏压缩": block-level
// statistics first, then the blocks to keep, without first assembling the dense matrix.  The
// sender's map is its causal attention distribution
//   A_s[i][j] = 2^(x_ij - lse_i),   x_ij = scale * log2(e) * q_{i,s} . k_{j,g},   j <= i < L,
//   lse_i = log2 sum_{j <= i} 2^x_ij,   g = floor(s * h_kv / h_s),
// so a block's mass needs, per row, the block's exp-sum and the row's lse.  Three passes:
//
//   k_qk<false> (stats)   item = (sequence, 128 query rows = two 64-row query blocks, head);
//                         for every causal 64-key block: S = Q K^T on the tensor cores
//                         (tcgen05, M=128 N=64 K=16 x 8, Q and K tiles by TMA, 128-byte
//                         swizzle, S double-buffered in TMEM), then one thread per row takes
//                         the block's max m and exp-sum l = sum 2^(x - m) (causal mask on the
//                         diagonal block), stores (m, l) and folds it into the row's running
//                         lse, stored once the item has walked all the row's blocks.
//   k_qk_mass             one CTA per causal block: the head-summed mass
//                         sum_{s, i} l 2^(m - lse) in float64, fixed order.  Selection and
//                         row_ptr / col_idx then run exactly as for dense maps.
//   k_qk<true> (gather)   the same item walk over the kept blocks of the item's two query
//                         blocks only (their ascending union): S recomputed, A = 2^(x - lse)
//                         written as bfloat16 values (0 where j > i or i >= L).
//
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer + TMEM owner, warps 2-5 one
// thread per query row (TMEM lane quarter warp % 4).  Three CTAs share an SM (a two-stage K
// ring keeps each within a third of the shared memory), so one CTA's exponentials overlap the
// others' MMAs.  Every mbarrier wait is bounded: on expiry the CTA
// records ST_TIMEOUT, every role stops, in-flight copies and MMAs are drained (bounded) and
// TMEM is freed.
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

constexpr int QT = 192;                        // 6 warps
constexpr int QROWS = 128;                     // query rows per item
constexpr int KB = 64;                         // keys per tile (= block size)
constexpr int DH = 128;                        // head dim
constexpr int KS = 2;                          // K ring stages
constexpr int CTAS_PER_SM = 3;                 // resident CTAs per SM (shared memory, TMEM, threads)
constexpr uint32_t Q_BYTES = QROWS * DH * 2;   // 32 KB: two 16 KB halves (dims 0-63, 64-127)
constexpr uint32_t K_BYTES = KB * DH * 2;      // 16 KB: two 8 KB halves
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_BAR = OFF_K + KS * K_BYTES;
constexpr uint32_t QK_SMEM = OFF_BAR + 256 + 1024;  // + alignment slack
constexpr int META_HDR = 4;                    // CompressWs::meta header words
enum {
  B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_KEMPTY = B_KFULL + KS, B_SFULL = B_KEMPTY + KS,
  B_SEMPTY = B_SFULL + 2, B_DONE = B_SEMPTY + 2,
  B_NEVER = B_DONE + 1,  // test stall: nothing ever arrives here
  B_COUNT = B_NEVER + 1
};
static_assert(B_COUNT * 8 <= 256, "barrier area");
static_assert(CTAS_PER_SM * QK_SMEM <= 232448, "CTAs per SM");
static_assert(CTAS_PER_SM * 128 <= 512, "TMEM columns of the resident CTAs");
// kind::f16, D float32, A and B bf16 K-major, N = 64, M = 128
constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) |
                              ((128u >> 4) << 24);

struct QkParams {
  const int64_t* meta;
  const int32_t* cu;
  int nseq, nqt_max, h_s, h_kv;
  int64_t n_items;
  float c2;                 // scale * log2(e)
  float2* ml;               // [h_s][cb_stride][64]: (m, l) of (head, causal block, row)
  int64_t cb_stride;
  float* lse2;              // [h_s][T]
  int64_t T;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t capacity;
  __nv_bfloat16* values;
  double* mass;
  uint32_t* status;
  uint64_t wait_ns;  // limit of every pipeline wait
  int stall;         // test: the MMA warp first waits on B_NEVER
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
__device__ __forceinline__ void bar_arrive(uint32_t b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
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
__device__ __forceinline__ void bar_drain(uint32_t b, uint32_t parity) {
  const uint64_t t0 = gtimer();
  while (!bar_try(b, parity) && gtimer() - t0 < DRAIN_NS) {}
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
// 2^x on the special-function unit (ex2.approx.ftz: results below 2^-126 flush to 0; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// K-major operand, 128-byte swizzle: 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t kmajor_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024u >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// 32 lanes x 32 columns of 32 bits; the wait and a register fence keep every use after it
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
}
__device__ __forceinline__ void ld_wait(uint32_t (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                 "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                 "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                 "+r"(v[30]), "+r"(v[31]));
}

// ------------------------------------------------------------------ work items and tiles
struct QItem {
  bool valid;
  int s, head, qt, L, nqb, qb0;
  int64_t t0, row0, cb0;  // first token, first BSR row, first causal block of the sequence
};

// item idx: the largest query tiles first (static striding then balances the CTAs), and
// within a tile index sequences then heads
__device__ __forceinline__ QItem qdecode(const QkParams& p, int64_t idx) {
  QItem it;
  const int64_t per = (int64_t)p.nseq * p.h_s;
  it.qt = p.nqt_max - 1 - (int)(idx / per);
  const int64_t r = idx - (idx / per) * per;
  it.s = (int)(r / p.h_s);
  it.head = (int)(r - (int64_t)it.s * p.h_s);
  const int64_t* m = p.meta + META_HDR + 4 * it.s;
  it.L = (int)m[0];
  it.nqb = (int)m[1];
  it.row0 = m[2];
  it.cb0 = m[3];
  it.t0 = p.cu[it.s];
  it.qb0 = 2 * it.qt;
  it.valid = it.qb0 < it.nqb;
  return it;
}

// the key blocks of an item, ascending: every causal block (stats), or the union of the kept
// blocks of its two query blocks with their BSR positions (gather; -1 where a row did not
// keep the block).  Every role walks the same sequence.
struct TileIt {
  int kb, kmax;               // stats
  int64_t p0, e0, p1, e1;     // gather cursors into col_idx
};
template <bool GATHER>
__device__ __forceinline__ void tiles_begin(const QkParams& p, const QItem& it, TileIt& t) {
  if (!GATHER) {
    t.kb = 0;
    t.kmax = min(it.qb0 + 1, it.nqb - 1);
  } else {
    const int64_t r0 = it.row0 + it.qb0;
    t.p0 = p.row_ptr[r0];
    t.e0 = min((int64_t)p.row_ptr[r0 + 1], p.capacity);
    if (it.qb0 + 1 < it.nqb) {
      t.p1 = p.row_ptr[r0 + 1];
      t.e1 = min((int64_t)p.row_ptr[r0 + 2], p.capacity);
    } else {
      t.p1 = t.e1 = 0;
    }
  }
}
template <bool GATHER>
__device__ __forceinline__ bool tiles_next(const QkParams& p, const QItem& it, TileIt& t, int* kb,
                                           int64_t* n0, int64_t* n1) {
  if (!GATHER) {
    if (t.kb > t.kmax) return false;
    *kb = t.kb++;
    *n0 = *n1 = -1;
    return true;
  }
  const int c0 = t.p0 < t.e0 ? p.col_idx[t.p0] : 0x7fffffff;
  const int c1 = t.p1 < t.e1 ? p.col_idx[t.p1] : 0x7fffffff;
  const int k = min(c0, c1);
  if (k == 0x7fffffff) return false;
  *n0 = c0 == k ? t.p0++ : -1;
  *n1 = c1 == k ? t.p1++ : -1;
  // a column outside the causal range of its row is never written by selection; skip it
  if (k < 0 || k > it.qb0 + 1) {
    *n0 = *n1 = -1;
    *kb = 0;
    return true;
  }
  if (k > it.qb0) *n0 = -1;
  *kb = k;
  return true;
}

// ------------------------------------------------------------------ stats / gather kernel
template <bool GATHER>
__global__ void __launch_bounds__(QT, CTAS_PER_SM)
    k_qk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ QkParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sb = su32(smem);
  auto bar = [&](int k) { return sb + OFF_BAR + 8u * (uint32_t)k; };
  const int gq = p.h_s / p.h_kv;

  if (threadIdx.x == 0) {
    s_abort = 0;
    bar_init(bar(B_QFULL), 1);
    bar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < KS; ++s) {
      bar_init(bar(B_KFULL + s), 1);
      bar_init(bar(B_KEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      bar_init(bar(B_SFULL + b), 1);
      bar_init(bar(B_SEMPTY + b), 4);
    }
    bar_init(bar(B_DONE), 1);
    bar_init(bar(B_NEVER), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(&s_tmem)),
                 "r"(128)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ================================================================ TMA producer
    // the whole warp waits (a warp waiting with all lanes is suspended by the hardware; a lone
    // polling lane would take issue slots from the row threads); lane 0 issues the copies
    bool ok = true;
    int64_t tc = 0, qi = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
      const QItem it = qdecode(p, idx);
      if (!it.valid) continue;
      TileIt ti;
      tiles_begin<GATHER>(p, it, ti);
      int kb;
      int64_t n0, n1;
      bool first = true;
      const int g = it.head / gq;
      while (ok && tiles_next<GATHER>(p, it, ti, &kb, &n0, &n1)) {
        if (first) {
          ok = __all_sync(0xffffffffu, bar_wait(bar(B_QEMPTY), (uint32_t)(qi & 1) ^ 1u, abort_flag,
                                                p.status, p.wait_ns));
          if (!ok) break;
          if (lane == 0) {
            bar_expect(bar(B_QFULL), Q_BYTES);
            const int row = (int)(it.t0 + (int64_t)QROWS * it.qt);
            tma3(sb + OFF_Q, &tmQ, bar(B_QFULL), 0, it.head, row);
            tma3(sb + OFF_Q + Q_BYTES / 2, &tmQ, bar(B_QFULL), 64, it.head, row);
          }
          __syncwarp();
          first = false;
          ++qi;
        }
        const int st = (int)(tc % KS);
        ok = __all_sync(0xffffffffu, bar_wait(bar(B_KEMPTY + st), (uint32_t)((tc / KS) & 1) ^ 1u,
                                              abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        if (lane == 0) {
          bar_expect(bar(B_KFULL + st), K_BYTES);
          const int key = (int)(it.t0 + (int64_t)KB * kb);
          tma3(sb + OFF_K + st * K_BYTES, &tmK, bar(B_KFULL + st), 0, g, key);
          tma3(sb + OFF_K + st * K_BYTES + K_BYTES / 2, &tmK, bar(B_KFULL + st), 64, g, key);
        }
        __syncwarp();
        ++tc;
      }
    }
    // drain: the last copies issued into every stage and into Q
    if (lane == 0) {
      for (int s = 0; s < KS; ++s) {
        const int64_t cnt = tc > s ? (tc - s - 1) / KS + 1 : 0;
        if (cnt) bar_drain(bar(B_KFULL + s), (uint32_t)((cnt - 1) & 1));
      }
      if (qi) bar_drain(bar(B_QFULL), (uint32_t)((qi - 1) & 1));
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issue
    bool ok = true;
    int64_t tc = 0, qi = 0;
    // test stall: a wait that can only run out (the whole CTA then stops as on any timeout)
    if (p.stall)
      ok = __all_sync(0xffffffffu, bar_wait(bar(B_NEVER), 0, abort_flag, p.status, p.wait_ns));
    for (int64_t idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
      const QItem it = qdecode(p, idx);
      if (!it.valid) continue;
      TileIt ti;
      tiles_begin<GATHER>(p, it, ti);
      int kb;
      int64_t n0, n1;
      bool first = true;
      while (ok && tiles_next<GATHER>(p, it, ti, &kb, &n0, &n1)) {
        if (first) {
          ok = __all_sync(0xffffffffu,
                          bar_wait(bar(B_QFULL), (uint32_t)(qi & 1), abort_flag, p.status, p.wait_ns));
          if (!ok) break;
          first = false;
        }
        const int st = (int)(tc % KS), b = (int)(tc & 1);
        ok = __all_sync(0xffffffffu, bar_wait(bar(B_KFULL + st), (uint32_t)((tc / KS) & 1),
                                              abort_flag, p.status, p.wait_ns));
        if (ok)
          ok = __all_sync(0xffffffffu, bar_wait(bar(B_SEMPTY + b), (uint32_t)((tc >> 1) & 1) ^ 1u,
                                                abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        if (lane == 0) {
          fence_after();
          const uint32_t qa = sb + OFF_Q, ka = sb + OFF_K + st * K_BYTES;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {  // 16 dims per MMA: +32 bytes in a half
            const uint64_t ad = kmajor_sw128(qa + (kk >> 2) * (Q_BYTES / 2)) + 2u * (kk & 3);
            const uint64_t bd = kmajor_sw128(ka + (kk >> 2) * (K_BYTES / 2)) + 2u * (kk & 3);
            mma(tmem + (uint32_t)(b * KB), ad, bd, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          commit(bar(B_KEMPTY + st));
          commit(bar(B_SFULL + b));
        }
        __syncwarp();
        ++tc;
      }
      if (!first) {
        if (lane == 0) commit(bar(B_QEMPTY));
        __syncwarp();
        ++qi;
      }
    }
    if (lane == 0) {
      commit(bar(B_DONE));
      bar_drain(bar(B_DONE), 0);
    }
    __syncwarp();
  } else {
    // ================================================================ one thread per row
    const int q = warp & 3, r = q * 32 + lane;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    bool ok = true;
    int64_t tc = 0;
    for (int64_t idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
      const QItem it = qdecode(p, idx);
      if (!it.valid) continue;
      const int i = QROWS * it.qt + r, qb = it.qb0 + (r >> 6), ii = r & 63;
      const bool row_ok = i < it.L && it.t0 + i < p.T;
      if (!GATHER && i < it.L && !row_ok) atomicOr(p.status, ST_INDEX);  // cu_seqlens past T
      float lse = 0.0f;
      if (GATHER && row_ok) lse = p.lse2[(int64_t)it.head * p.T + it.t0 + i];
      float run_m = -INFINITY, run_s = 0.0f;  // stats: the row's running max and exp-sum
      TileIt ti;
      tiles_begin<GATHER>(p, it, ti);
      int kb;
      int64_t n0, n1;
      while (tiles_next<GATHER>(p, it, ti, &kb, &n0, &n1)) {
        const int b = (int)(tc & 1);
        ok = __all_sync(0xffffffffu, bar_wait(bar(B_SFULL + b), (uint32_t)((tc >> 1) & 1),
                                              abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        fence_after();
        uint32_t v0[32], v1[32];
        ld32(trow + (uint32_t)(b * KB), v0);
        ld32(trow + (uint32_t)(b * KB + 32), v1);
        ld_wait(v0);
        ld_wait(v1);
        fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(bar(B_SEMPTY + b));
        ++tc;
        const bool diag = kb == qb;
        float sv[64];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sv[c] = __uint_as_float(v0[c]);
          sv[c + 32] = __uint_as_float(v1[c]);
        }
        if (diag || !row_ok) {  // keys j > i (and every key of a row past the sequence) drop out
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!row_ok || c > ii) sv[c] = -INFINITY;
        }
        if (!GATHER) {
          if (row_ok && kb <= qb) {
            // max of the raw scores (scaling by c2 > 0 keeps the order), eight chains
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = sv[k];
#pragma unroll
            for (int c = 8; c < 64; ++c) m8[c & 7] = fmaxf(m8[c & 7], sv[c]);
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * p.c2;
            float l8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) l8[k] = 0.0f;
#pragma unroll
            for (int c = 0; c < 64; ++c) l8[c & 7] += ex2(fmaf(sv[c], p.c2, -mx));
            const float l = ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
            const int64_t cb = it.cb0 + (int64_t)qb * (qb + 1) / 2 + kb;
            p.ml[((int64_t)it.head * p.cb_stride + cb) * KB + ii] = make_float2(mx, l);
            const float nm = fmaxf(run_m, mx);
            run_s = run_s * ex2(run_m - nm) + l * ex2(mx - nm);
            run_m = nm;
          }
        } else {
          const int64_t n = r < 64 ? n0 : n1;
          if (n >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.values + (((int64_t)n * p.h_s + it.head) * KB + ii) * KB);
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = 8 * c8 + 2 * e;
                const __nv_bfloat162 pk = __floats2bfloat162_rn(ex2(fmaf(sv[c], p.c2, -lse)),
                                                                ex2(fmaf(sv[c + 1], p.c2, -lse)));
                w[e] = *reinterpret_cast<const uint32_t*>(&pk);
              }
              dst[c8] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      // the item walked every causal key block of its rows: the row's log2-sum-exp
      if (!GATHER && ok && row_ok) p.lse2[(int64_t)it.head * p.T + it.t0 + i] = run_m + log2f(run_s);
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

// ------------------------------------------------------------------ masses
__device__ inline int find_cb_seq(const int64_t* meta, int nseq, int64_t cb) {
  int lo = 0, hi = nseq - 1;  // last s whose first causal block is <= cb
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (meta[META_HDR + 4 * mid + 3] <= cb) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ inline int tri_row_of(int64_t c) {  // q with q (q + 1) / 2 <= c < (q + 1) (q + 2) / 2
  int q = (int)((sqrt(8.0 * (double)c + 1.0) - 1.0) * 0.5);
  while ((int64_t)(q + 1) * (q + 2) / 2 <= c) ++q;
  while ((int64_t)q * (q + 1) / 2 > c) --q;
  return q;
}

// One CTA per causal block (qb, kb): mass = sum over heads s and rows i of the block of
// l 2^(m - lse_i), float64; each thread sums its (head, row) pairs in a fixed order, then a
// fixed shuffle tree and a fixed pass over the warps.
constexpr int RT = 256;
__global__ void __launch_bounds__(RT) k_qk_mass(const __grid_constant__ QkParams p) {
  __shared__ double red[RT / 32];
  const int64_t cb = blockIdx.x;
  if (cb >= p.meta[1]) return;
  const int s = find_cb_seq(p.meta, p.nseq, cb);
  const int64_t* m = p.meta + META_HDR + 4 * s;
  const int L = (int)m[0];
  const int64_t c = cb - m[3];
  const int qb = tri_row_of(c);
  const int64_t t0 = p.cu[s] + (int64_t)KB * qb;
  const int nv = min(KB, L - KB * qb);
  // warp w takes heads w, w + 8, ...; lane l rows 2l and 2l + 1 (one 16-byte load of the two
  // (m, l) pairs); the loop is unrolled so several heads' loads are in flight
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = 2 * lane;
  double acc = 0.0;
  if (t0 + nv > p.T) {  // cu_seqlens past T: reported by the stats pass
    if (threadIdx.x == 0) p.mass[cb] = 0.0;
    return;
  }
#pragma unroll 4
  for (int hs = warp; hs < p.h_s; hs += RT / 32) {
    const float4 v = *reinterpret_cast<const float4*>(p.ml + ((int64_t)hs * p.cb_stride + cb) * KB + i0);
    const float* lr = p.lse2 + (int64_t)hs * p.T + t0;
    if (i0 < nv) acc += (double)v.y * (double)ex2(v.x - lr[i0]);
    if (i0 + 1 < nv) acc += (double)v.w * (double)ex2(v.z - lr[i0 + 1]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < RT / 32; ++w) t += red[w];
    p.mass[cb] = t;
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// [T][h][128] bf16 -> dims (dim, head, token), box (64, 1, rows), 128-byte swizzle
bool encode_qk(CUtensorMap* tm, const void* base, int h, int64_t T, uint32_t rows,
               std::string* err) {
  auto fn = get_encode();
  if (!fn) { *err = "cuTensorMapEncodeTiled unavailable"; return false; }
  const uint64_t dims[3] = {(uint64_t)DH, (uint64_t)h, (uint64_t)std::max<int64_t>(T, 1)};
  const uint64_t strides[2] = {(uint64_t)DH * 2, (uint64_t)h * DH * 2};
  const uint32_t box[3] = {64, 1, rows};
  const uint32_t es[3] = {1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { *err = "cuTensorMapEncodeTiled failed: " + std::to_string((int)r); return false; }
  return true;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

mf_compress_desc base_desc(const mf_compress_qk_desc& d) {
  mf_compress_desc c{};
  c.nseq = d.nseq;
  c.max_seqlen = d.max_seqlen;
  c.B = d.B;
  c.capacity_blocks = d.capacity_blocks;
  c.h_s = d.h_s;
  return c;
}

}  // namespace

size_t compress_qk_ws_layout(const mf_compress_qk_desc& d, CompressWs* ws, QkWs* q, void* base) {
  const mf_compress_desc c = base_desc(d);
  size_t off = align_up(compress_ws_layout(c, ws, base), 256);
  const int64_t nqb_max = (d.max_seqlen + d.B - 1) / d.B;
  const int64_t max_cb = (int64_t)d.nseq * nqb_max * (nqb_max + 1) / 2;
  const size_t o_ml = off;
  off = align_up(off + sizeof(float2) * (size_t)d.h_s * (size_t)max_cb * KB, 256);
  const size_t o_lse = off;
  off = align_up(off + sizeof(float) * (size_t)d.h_s * (size_t)std::max<int64_t>(d.T, 1), 256);
  if (q) {
    char* b = static_cast<char*>(base);
    q->ml = reinterpret_cast<float2*>(b + o_ml);
    q->lse2 = reinterpret_cast<float*>(b + o_lse);
    q->cb_stride = max_cb;
  }
  return off;
}

bool launch_compress_qk(const mf_compress_qk_desc& d, const CompressWs& ws, const QkWs& q,
                        uint32_t* status, cudaStream_t st, std::string* err) {
  cudaError_t e = launch_meta(d.cu_seqlens, nullptr, d.nseq, d.max_seqlen, d.B, 2, ws, status,
                              d.row_ptr, d.nnz_out, st);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  if (d.max_seqlen == 0) return true;  // no query block: k_meta wrote the empty BSR
  CUtensorMap tmQ, tmK;
  if (!encode_qk(&tmQ, d.Q, d.h_s, d.T, QROWS, err)) return false;
  if (!encode_qk(&tmK, d.K, d.h_kv, d.T, KB, err)) return false;
  QkParams p{};
  p.meta = ws.meta;
  p.cu = d.cu_seqlens;
  p.nseq = d.nseq;
  p.nqt_max = (d.max_seqlen + QROWS - 1) / QROWS;
  p.h_s = d.h_s;
  p.h_kv = d.h_kv;
  p.n_items = (int64_t)p.nqt_max * d.nseq * d.h_s;
  const double scale = d.scale > 0.0f ? (double)d.scale : 1.0 / std::sqrt((double)d.d);
  p.c2 = (float)(scale * 1.4426950408889634);  // log2(e)
  p.ml = q.ml;
  p.cb_stride = q.cb_stride;
  p.lse2 = d.lse_out ? d.lse_out : q.lse2;
  p.T = d.T;
  p.row_ptr = d.row_ptr;
  p.col_idx = d.col_idx;
  p.capacity = d.capacity_blocks;
  p.values = static_cast<__nv_bfloat16*>(d.values);
  p.mass = d.block_mass_out ? d.block_mass_out : ws.mass;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  p.stall = wait_stall();
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(p.n_items, CTAS_PER_SM * (int64_t)sms));
  e = cudaFuncSetAttribute(k_qk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QK_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_qk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QK_SMEM);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  // 1. (m, l) of every (head, causal block, row)
  k_qk<false><<<grid, QT, QK_SMEM, st>>>(tmQ, tmK, p);
  // 2. masses of every causal block, then selection
  k_qk_mass<<<(unsigned)ws.max_cb, RT, 0, st>>>(p);
  e = launch_select(ws, d.nseq, d.max_seqlen, d.B, p.mass, d.tau, d.row_ptr, d.col_idx, d.nnz_out,
                    d.capacity_blocks, status, st);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  // 3. the kept blocks' values
  k_qk<true><<<grid, QT, QK_SMEM, st>>>(tmQ, tmK, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  return true;
}

}  // namespace mfi
