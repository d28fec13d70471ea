// Fused map retrieval on sm_100a tensor cores: clusters of four CTAs (tcgen05 + TMA + TMEM +
// distributed shared memory).
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com),
// section "存不下、读得慢?三个工程优化手段", subsection 3 "算得省的:融合内核执行":
// read the kept sparse blocks, mix sender heads into receiver heads on chip,
// multiply by the receiver's V and accumulate, without materialising the
// receiver's dense map.  The pages' kernel is Triton on A800; this one is a
// new design for B200.
//
// Work unit = (sequence, query block, 32-row window, head chunk of 8 KV groups x 4 virtual
// receiver heads; a group of gq <= 4 heads is padded to 4).  One cluster of four CTAs takes a
// unit at a time (persistent: the clusters walk the units, largest query blocks first); every
// CTA of the cluster walks the same units and tiles.  CTA k of the cluster, for each kept
// 64-key tile of the unit:
//
//   mixing   D1[pos][(part, v)] = sum_s A_s[pos] W_part[v][s]      tcgen05 M=128 N=64 K=16
//            for its own 8 rows [8k, 8k+8) of the window and all 32 virtual heads:
//            pos = (row, key) of 2 rows x 64 keys (4 M tiles), A MN-major SW128 straight from
//            TMA; W split into bf16 hi and lo parts stacked along N (~16 bits of W);
//   convert  P = hi + lo (float32), causal mask, P rounded to float16; the part of each KV
//            group is sent to the CTA that owns the group (CTA g owns groups 2g, 2g+1 of the
//            chunk) with st.async into its shared memory, completing bytes on its barrier;
//   P.V      for its two groups and all 32 rows of the window, D2 in TMEM:
//            D2[dim][(row, head)] += V^T[dim][key] P^T[key][(row, head)]   M=128 N=128 K=16,
//            float16 operands, float32 accumulation; V of the group is read from global
//            memory by four loader warps, converted bf16 -> float16 (exact within the float16
//            range) and stored in the MN-major SW128 operand layout;
//   epilogue once the unit's last tile is done: D2 rounded to bf16 and stored as O rows.
// So every kept map tile is read once from HBM, the mixing has every receiver head in one
// MMA, and P.V runs at N = 128 with V read once per 32 rows.  A P.V commit is multicast to
// all four CTAs' "P slot free" barriers; the owner of a slot announces the bytes it expects.
//
// Arithmetic: W ~16 bits (hi + lo bf16), P float32 rounded to float16 (relative 2^-11), V
// float16 (exact for |V| <= 65504), float32 accumulation, O rounded to bf16.  A |V| or |P|
// above the float16 range sets status bit ST_RANGE.
//
// Warp roles (12 warps): 0 TMA producer of the map tiles; 1 mixing MMA issuer + TMEM owner;
// 2 P.V MMA issuer; 3 idle; 4-7 converters (one per TMEM lane quarter) and the O epilogue;
// 8-11 V loaders.  TMEM: D2 (two groups x 128 columns) in [0, 256), D1 (4 M tiles x 64
// columns, two halves with their own barriers) in [256, 512).  Every mbarrier wait is bounded
// (mf_set_wait_limit, default 2 s): on expiry the CTA records ST_TIMEOUT and every role
// stops; issued copies and MMAs are drained (bounded), the cluster meets once more so that no
// CTA leaves while a peer may still write into it, and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "mf_internal.cuh"

namespace mfi {
namespace {

constexpr int CS = 4;             // CTAs per cluster
constexpr int WR = 32;            // query rows per unit
constexpr int RM = WR / CS;       // rows mixed by each CTA: 8
constexpr int KT = 64;            // keys per tile
constexpr int NGC = 8;            // KV groups per head chunk
constexpr int GO = NGC / CS;      // groups owned by each CTA: 2
constexpr int GQP = 4;            // virtual heads per group
constexpr int HV = NGC * GQP;     // virtual heads per chunk: 32
constexpr int D = 128;            // head dim
constexpr int SC = 16;            // sender heads per A chunk (one MMA K step)
constexpr int NPV = WR * GQP;     // P.V N of one group: 128
constexpr int NT = 384;           // 12 warps
constexpr int A_STAGES = 4;       // >= sender-head chunks of a tile (h_s <= 64)
constexpr int PSLOTS = 2, VSLOTS = 2;
constexpr uint32_t A_BYTES = RM * SC * KT * 2;     // 16 KB: 8 rows x 16 heads x 64 keys
constexpr uint32_t PG_BYTES = NPV * KT * 2;        // 16 KB: one group's P^T of a tile
constexpr uint32_t PSLOT_BYTES = GO * PG_BYTES;    // 32 KB
constexpr uint32_t VG_BYTES = D * KT * 2;          // 16 KB: one group's V tile
constexpr uint32_t VSLOT_BYTES = GO * VG_BYTES;    // 32 KB
constexpr uint32_t W_CHUNK = 2 * HV * SC * 2;      // 2 KB: W^T (hi and lo rows) of 16 sender heads
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_P = OFF_A + A_STAGES * A_BYTES;
constexpr uint32_t OFF_V = OFF_P + PSLOTS * PSLOT_BYTES;
constexpr uint32_t OFF_W = OFF_V + VSLOTS * VSLOT_BYTES;
constexpr int ITEMS_MAX = 32;                      // units per CTA decoded up front
constexpr uint32_t ITEM_BYTES = 64;
constexpr uint32_t OFF_ITEMS = OFF_W + 4 * W_CHUNK;
constexpr uint32_t OFF_BAR = OFF_ITEMS + ITEMS_MAX * ITEM_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory of one CTA");
static_assert(OFF_P % 1024 == 0 && OFF_V % 1024 == 0 && OFF_W % 1024 == 0, "operand alignment");
constexpr float F16_MAX = 65504.0f;
constexpr uint64_t GRACE_NS = 100000;  // after an abort: time for peers' stores still in flight

// barrier slots (8 bytes each)
enum {
  B_AFULL = 0, B_AEMPTY = B_AFULL + A_STAGES,
  B_D1FULL = B_AEMPTY + A_STAGES,  // [2]: halves of D1 (M tiles 0-1, 2-3)
  B_D1EMPTY = B_D1FULL + 2,        // [2]
  B_PFULL = B_D1EMPTY + 2,         // [PSLOTS]: st.async bytes of all four CTAs + the owner's expect
  B_PEMPTY = B_PFULL + PSLOTS,     // [PSLOTS]: P.V commits of the four owners (multicast)
  B_VFULL = B_PEMPTY + PSLOTS,     // [VSLOTS]: the four V loader warps
  B_VEMPTY = B_VFULL + VSLOTS,     // [VSLOTS]: this CTA's P.V commit
  B_OFULL = B_VEMPTY + VSLOTS,     // D2 of a unit complete
  B_OEMPTY = B_OFULL + 1,          // [GO]: a group's D2 read by the epilogue
  B_DRAIN1 = B_OEMPTY + GO, B_DRAIN2 = B_DRAIN1 + 1,
  B_NEVER = B_DRAIN2 + 1,          // test stall: nothing ever arrives here
  B_COUNT = B_NEVER + 1
};
static_assert(B_COUNT * 8 <= 512, "barrier area");

// instruction descriptors (kind::f16): D f32 (bit 4), A / B type at bits 7 / 10 (0 f16,
// 1 bf16), A / B major at bits 15 / 16 (1 = MN-major), N >> 3 at bit 17, M >> 4 at bit 24
constexpr uint32_t IDESC_MIX = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (0u << 16) |
                               ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t IDESC_PV = (1u << 4) | (0u << 7) | (0u << 10) | (1u << 15) | (1u << 16) |
                              ((128u >> 3) << 17) | ((128u >> 4) << 24);

constexpr int NRMAX = 4;  // receivers served by one launch (one BSR, several W / V / O)

// one receiver: its head map, V and O (and its V paging)
struct RecvParams {
  const float* W;  // [h_r][h_s]
  void* O;         // bf16, or float32 when o_f32
  int o_f32;
  const __nv_bfloat16* V;
  const int32_t* block_table;
  int paged, page_size, n_pages, max_pages;
  int64_t total_k;  // rows of a contiguous V
  int h_r, h_kv, gq, hcs;
};
struct TcParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t capacity;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* qblock_base;
  int nseq, nqbq, wcs;     // sequences, query blocks per sequence (bound), windows per block
  int NH;                  // head chunks of all receivers together
  int hh_base[NRMAX + 1];  // first head chunk of each receiver
  int nrecv;
  int n_units;
  int h_s, nsc, B;
  RecvParams rv[NRMAX];
  uint32_t* status;
  uint64_t wait_ns;  // limit of every pipeline wait
  int stall;         // test: the mixing issuer first waits on B_NEVER
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
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
// try_wait; with CL, cluster-scope acquire (for the barriers peer CTAs signal: data a peer
// wrote before completing the phase is visible once it returns true)
template <bool CL = false>
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  if (CL)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
  return ok != 0;
}
// Bounded wait: false if the CTA aborted or the wait ran out of time (limit_ns).
template <bool CL = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint64_t limit_ns) {
  if (mbar_try<CL>(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try<CL>(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(status, ST_TIMEOUT);
        return false;
      }
    }
  }
}
template <bool CL = false>
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try<CL>(bar, parity) && globaltimer() - t0 < DRAIN_NS) {}
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_map(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// 16 bytes into a peer CTA's shared memory, completing 16 bytes on its barrier
__device__ __forceinline__ void st_async16(uint32_t raddr, uint32_t rbar, uint32_t a, uint32_t b,
                                           uint32_t c, uint32_t d) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(raddr), "r"(a), "r"(b), "r"(c), "r"(d), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// commit whose barrier arrival goes to the barrier at the same offset in every CTA of `mask`
__device__ __forceinline__ void tc_commit_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// shared-memory matrix descriptor: start, leading/stride byte offsets, SM100 version bit,
// layout (0 = no swizzle, 2 = 128-byte swizzle)
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
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
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Register fence: the compiler sees v redefined here, so no use of v moves above this point
// (above the tcgen05.wait::ld that makes v valid).
__device__ __forceinline__ void reg_fence(uint32_t (&v)[32]) {
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                 "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                 "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                 "+r"(v[30]), "+r"(v[31]));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// two bf16 (one 32-bit word) -> two float16 (one word); |x| is folded into amax
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t w, float& amax) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xFFFF0000u);
  amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
  return pack_h2(a, b);
}

// ------------------------------------------------------------------ work units
struct Unit {
  int s, qb, i_begin, row_lo, row_hi, k_len, n_tiles, k0, kb0;
  int64_t rp0;
  int64_t o_row0;  // O row of window row 0 (cu_seqlens_q[s] + i_begin - q0)
  bool valid, bsr_ok;
};
static_assert(sizeof(Unit) <= ITEM_BYTES, "unit table slot");

// unit idx = ((qbr * nseq + s) * wcs + w) * NH + hh: qbr counts query blocks back from the
// last one of the sequence's chunk, so the largest units (most kept blocks) come first;
// hh = a receiver's head chunk.  Identical in every role and every CTA of the cluster.
__device__ __forceinline__ Unit decode(const TcParams& p, int idx) {
  Unit u;
  u.valid = false;
  u.bsr_ok = true;
  u.n_tiles = 0;
  idx /= p.NH;
  const int w = idx % p.wcs;
  idx /= p.wcs;
  const int s = idx % p.nseq;
  const int qbr = idx / p.nseq;
  const int q_len = p.cu_q[s + 1] - p.cu_q[s];
  const int k_len = p.cu_k[s + 1] - p.cu_k[s];
  const int q0 = k_len - q_len;
  if (q_len <= 0 || q0 < 0) return u;
  const int qb_first = q0 / p.B, qb_last = (k_len - 1) / p.B;
  const int qb = qb_last - qbr;
  if (qb < qb_first) return u;
  const int i_begin = qb * p.B + w * WR;
  const int row_lo = max(q0, i_begin), row_hi = min(k_len, i_begin + WR);
  if (row_lo >= row_hi) return u;
  const int64_t brow = (int64_t)p.qblock_base[s] + qb;
  const int64_t rp0 = p.row_ptr[brow], rp1 = p.row_ptr[brow + 1];
  u.bsr_ok = rp0 >= 0 && rp1 >= rp0 && rp1 <= p.capacity && rp1 - rp0 <= qb + 1;
  u.n_tiles = u.bsr_ok ? (int)(rp1 - rp0) * (p.B / KT) : 0;
  u.s = s; u.qb = qb; u.i_begin = i_begin; u.row_lo = row_lo; u.row_hi = row_hi;
  u.k_len = k_len; u.rp0 = rp0; u.k0 = p.cu_k[s];
  u.kb0 = u.n_tiles > 0 ? p.col_idx[rp0] : -1;
  u.o_row0 = (int64_t)p.cu_q[s] + (i_begin - q0);
  u.valid = true;
  return u;
}

// Optional timeline trace (compile with -DMF_TRACE): for the first TRACE_CTAS CTAs, per role,
// SM-clock stamps of pipeline events kept in shared memory and copied out at the end, read back
// with mf_trace_dump().  Each role has a single writing thread.  Roles: 0 map producer, 1 mixing
// issuer, 2 P.V issuer, 3 first converter warp, 4 first V loader warp.
#ifdef MF_TRACE
constexpr int TRACE_CTAS = 16, TRACE_N = 512, TRACE_ROLES = 5;
__device__ uint64_t g_trace[TRACE_CTAS][TRACE_ROLES][TRACE_N];
#define TRACE(role, code)                                                                  \
  do {                                                                                     \
    const int n_ = s_tn[role];                                                             \
    if (n_ < TRACE_N - 1) {                                                                \
      s_tr[role][1 + n_] = ((uint64_t)(code) << 56) | ((uint64_t)clock64() & ((1ull << 56) - 1)); \
      s_tn[role] = n_ + 1;                                                                 \
    }                                                                                      \
  } while (0)
#else
#define TRACE(role, code)
#endif

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(NT, 1)
    k_retrieve_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
#ifdef MF_TRACE
  __shared__ uint64_t s_tr[TRACE_ROLES][TRACE_N];
  __shared__ volatile int s_tn[TRACE_ROLES];
  if (threadIdx.x < TRACE_ROLES) s_tn[threadIdx.x] = 0;
#endif
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)(blockIdx.x % CS);     // rank in the cluster (cluster dims (4, 1, 1))
  const int cl = (int)(blockIdx.x / CS), ncl = (int)(gridDim.x / CS);
  // receiver and head chunk: constant per cluster (the cluster count is a multiple of NH)
  const int hh = cl % p.NH;
  int ri = 0;
  while (ri + 1 < p.nrecv && hh >= p.hh_base[ri + 1]) ++ri;
  const RecvParams& q_r = p.rv[ri];
  const int hc = hh - p.hh_base[ri];
  const int tpb = p.B / KT;

  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + OFF_BAR;
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  // unit k of this cluster (idx = cl + k * ncl): the first ITEMS_MAX from the table decoded
  // once below, later ones decoded where they are needed
  Unit* s_units = reinterpret_cast<Unit*>(smem + OFF_ITEMS);
  auto unit = [&](int k, int idx) -> Unit { return k < ITEMS_MAX ? s_units[k] : decode(p, idx); };

  // ---- setup
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int k = 0; k < A_STAGES; ++k) { mbar_init(bar(B_AFULL + k), 1); mbar_init(bar(B_AEMPTY + k), 1); }
    for (int h = 0; h < 2; ++h) { mbar_init(bar(B_D1FULL + h), 1); mbar_init(bar(B_D1EMPTY + h), 4); }
    for (int k = 0; k < PSLOTS; ++k) { mbar_init(bar(B_PFULL + k), 1); mbar_init(bar(B_PEMPTY + k), CS); }
    for (int k = 0; k < VSLOTS; ++k) { mbar_init(bar(B_VFULL + k), 4); mbar_init(bar(B_VEMPTY + k), 1); }
    mbar_init(bar(B_OFULL), 1);
    for (int g = 0; g < GO; ++g) mbar_init(bar(B_OEMPTY + g), 4);
    mbar_init(bar(B_DRAIN1), 1);
    mbar_init(bar(B_DRAIN2), 1);
    mbar_init(bar(B_NEVER), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // W^T of this chunk's 32 virtual heads, bf16, K-major without swizzle, 64 rows per s:
  // row n < 32 is the hi part of virtual head n, row 32 + n its lo part.  Element (n, s) at
  // (s/8)*1024 + (n/8)*128 + (n%8)*16 + (s%8)*2.
  {
    const int ks = p.nsc * SC;
    uint16_t* wt = reinterpret_cast<uint16_t*>(smem + OFF_W);
    for (int e = threadIdx.x; e < HV * ks; e += NT) {
      const int v = e / ks, hs = e % ks;
      const int G = hc * NGC + v / GQP, q = v % GQP;
      float w = 0.0f;
      if (q < q_r.gq && G < q_r.h_kv && hs < p.h_s) w = q_r.W[(int64_t)(G * q_r.gq + q) * p.h_s + hs];
      __nv_bfloat16 hi = __float2bfloat16_rn(w);
      __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const int base = (hs >> 3) * 1024 + (hs & 7) * 2;
      wt[(base + (v >> 3) * 128 + (v & 7) * 16) >> 1] = *reinterpret_cast<uint16_t*>(&hi);
      wt[(base + ((v + HV) >> 3) * 128 + (v & 7) * 16) >> 1] = *reinterpret_cast<uint16_t*>(&lo);
    }
  }
  for (int k = threadIdx.x; k < ITEMS_MAX; k += NT) {
    const int idx = cl + k * ncl;
    if (idx < p.n_units) s_units[k] = decode(p, idx);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  // every CTA of the cluster has initialised its barriers before any peer signals them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ================================================================ TMA producer (map tiles)
    // the whole warp waits (suspended by the hardware); lane 0 issues the copies
    int as = 0;
    uint32_t aph = 0;
    int a_issued = 0;
    bool ok = true;
    for (int idx = cl, ik = 0; idx < p.n_units && ok; idx += ncl, ++ik) {
      const Unit u = unit(ik, idx);
      if (!u.valid) continue;
      if (!u.bsr_ok && rank == 0 && lane == 0) atomicOr(p.status, ST_INDEX);
      const int w = (idx / p.NH) % p.wcs;
      for (int t = 0; t < u.n_tiles && ok; ++t) {
        const int64_t e = u.rp0 + t / tpb;
        const int half = t % tpb;
        for (int c = 0; c < p.nsc && ok; ++c) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_AEMPTY + as), aph ^ 1, abort_flag, p.status, p.wait_ns));
          if (!ok) break;
          if (lane == 0) {
            TRACE(0, 1);
            mbar_expect_tx(bar(B_AFULL + as), A_BYTES);
            tma_load_4d(sb + OFF_A + as * A_BYTES, &tmA, bar(B_AFULL + as), half * KT, c * SC,
                        w * WR + rank * RM, (int)e);
          }
          __syncwarp();
          ++a_issued;
          if (++as == A_STAGES) { as = 0; aph ^= 1; }
        }
      }
    }
    // drain: wait (bounded) for the last copy issued into every stage
    if (lane == 0)
      for (int k = 0; k < A_STAGES; ++k) {
        const int cnt = a_issued > k ? (a_issued - k - 1) / A_STAGES + 1 : 0;
        if (cnt) mbar_drain(bar(B_AFULL + k), (cnt - 1) & 1);
      }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ mixing MMA issuer
    bool ok = true;
    // test stall: a wait that can only run out (the whole cluster then stops as on any timeout)
    if (p.stall) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_NEVER), 0, abort_flag, p.status, p.wait_ns));
    int as = 0;
    uint32_t aph = 0;
    int T = 0;  // tiles processed so far
    const uint64_t wdesc0 = smem_desc(sb + OFF_W, 1024u, 128u, 0u);
    const uint64_t adesc0 = smem_desc(sb + OFF_A, 2048u, 1024u, 2u);
    for (int idx = cl, ik = 0; idx < p.n_units && ok; idx += ncl, ++ik) {
      const Unit u = unit(ik, idx);
      if (!u.valid) continue;
      for (int t = 0; t < u.n_tiles && ok; ++t, ++T) {
        // half 0 (M tiles 0, 1) over all sender-head chunks, then half 1 (M tiles 2, 3); the
        // tile's chunks stay in the A ring until half 1 has read them (A_STAGES >= chunks)
        for (int hf = 0; hf < 2 && ok; ++hf) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_D1EMPTY + hf), (T & 1) ^ 1, abort_flag, p.status, p.wait_ns));
          if (!ok) break;
          if (lane == 0) TRACE(1, 2 + hf);
          int st = as;
          uint32_t ph = aph;
          for (int c = 0; c < p.nsc && ok; ++c) {
            if (hf == 0) {
              ok = __all_sync(0xffffffffu, mbar_wait(bar(B_AFULL + st), ph, abort_flag, p.status, p.wait_ns));
              if (!ok) break;
              if (lane == 0) TRACE(1, 4);
            }
            if (lane == 0) {
              tc_fence_after();
              const uint64_t ad = adesc0 + (((uint32_t)st * A_BYTES) >> 4);
              const uint64_t wd = wdesc0 + ((c * W_CHUNK) >> 4);
#pragma unroll
              for (int mm = 0; mm < 2; ++mm) {
                const int m = 2 * hf + mm;
                tc_mma(tmem + 256u + 64u * (uint32_t)m, ad + ((m * 4096u) >> 4), wd, IDESC_MIX,
                       c > 0 ? 1u : 0u);
              }
              if (hf == 1) tc_commit(bar(B_AEMPTY + st));
            }
            __syncwarp();
            if (++st == A_STAGES) { st = 0; ph ^= 1; }
          }
          if (!ok) break;
          if (lane == 0) tc_commit(bar(B_D1FULL + hf));
          __syncwarp();
          if (hf == 1) { as = st; aph = ph; }
        }
      }
    }
    if (lane == 0) {
      tc_commit(bar(B_DRAIN1));
      mbar_drain(bar(B_DRAIN1), 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ================================================================ P.V MMA issuer
    bool ok = true;
    int T = 0, K = 0;  // tiles and units processed so far
    const uint64_t vdesc0 = smem_desc(sb + OFF_V, 8192u, 1024u, 2u);
    const uint64_t pdesc0 = smem_desc(sb + OFF_P, 8192u, 1024u, 2u);
    int ng = 0;  // this CTA's real groups
    for (int gl = 0; gl < GO; ++gl) ng += (hc * NGC + rank * GO + gl < q_r.h_kv) ? 1 : 0;
    for (int idx = cl, ik = 0; idx < p.n_units && ok; idx += ncl, ++ik) {
      const Unit u = unit(ik, idx);
      if (!u.valid) continue;
      for (int t = 0; t < u.n_tiles && ok; ++t, ++T) {
        const int ps = T % PSLOTS, vs = T % VSLOTS;
        // the owner announces the bytes its peers will complete on the slot's barrier
        if (lane == 0) mbar_expect_tx(bar(B_PFULL + ps), PSLOT_BYTES);
        __syncwarp();
        if (lane == 0) TRACE(2, 5);
        ok = __all_sync(0xffffffffu, mbar_wait<true>(bar(B_PFULL + ps), (T / PSLOTS) & 1, abort_flag, p.status, p.wait_ns));
        if (lane == 0) TRACE(2, 6);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_VFULL + vs), (T / VSLOTS) & 1, abort_flag, p.status, p.wait_ns));
        if (lane == 0) TRACE(2, 7);
        // the previous unit's epilogue must have read D2 out
        for (int gl = 0; gl < GO && ok && t == 0 && K > 0; ++gl)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OEMPTY + gl), (K - 1) & 1, abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        if (lane == 0) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          tc_fence_after();
          for (int gl = 0; gl < ng; ++gl) {
            const uint64_t vd = vdesc0 + ((vs * VSLOT_BYTES + gl * VG_BYTES) >> 4);
            const uint64_t pd = pdesc0 + ((ps * PSLOT_BYTES + gl * PG_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < KT / 16; ++kk)
              tc_mma(tmem + 128u * (uint32_t)gl, vd + ((kk * 2048u) >> 4), pd + ((kk * 2048u) >> 4),
                     IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(B_VEMPTY + vs));
          tc_commit_mc(bar(B_PEMPTY + ps), (uint16_t)((1u << CS) - 1u));  // the slot is free in all four CTAs
          TRACE(2, 8);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (u.n_tiles == 0 && K > 0) {  // take the epilogue's phases in order all the same
        for (int gl = 0; gl < GO && ok; ++gl)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OEMPTY + gl), (K - 1) & 1, abort_flag, p.status, p.wait_ns));
        if (!ok) break;
      }
      if (lane == 0) tc_commit(bar(B_OFULL));  // D2 of this unit complete (at once with no tile)
      __syncwarp();
      ++K;
    }
    if (lane == 0) {
      tc_commit(bar(B_DRAIN2));
      mbar_drain(bar(B_DRAIN2), 0);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ================================================================ convert P, epilogue
    // Warp q owns TMEM lane quarter q: in every M tile its lane is position l = 32q + lane =
    // (row 2m + rb, key j) with j = l % 64, rb = l / 64.  Rows 2m + rb of the pair of M tiles
    // (0, 1) or (2, 3) at key j, 4 heads of a group each, make one 16-byte chunk of that
    // group's P^T: n = 8c + 4p + h with c = 4 rank + 2 pair + rb, p = row within the pair.
    const int q = warp & 3;
    const int l = q * 32 + lane;
    const int j = l & 63, rb = l >> 6;
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    // peers' shared-memory windows
    uint32_t rbase[CS];
#pragma unroll
    for (int r = 0; r < CS; ++r) rbase[r] = cluster_map(sb, (uint32_t)r);
    const int64_t rs = (int64_t)q_r.h_r * D;  // O row stride
    const int d = q * 32 + lane;               // epilogue: this lane's head dim
    // epilogue of a unit: D2 group gl -> O rows (bf16), lanes paired so that each store
    // writes two adjacent head dims
    auto epilogue = [&](int ek, int eidx, int Ke) -> bool {
      const Unit u = unit(ek, eidx);
      const bool have = u.n_tiles > 0;
      const int ilo = u.row_lo - u.i_begin, ihi = u.row_hi - u.i_begin;
      if (warp == 4 && lane == 0) TRACE(3, 15);
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), Ke & 1, abort_flag, p.status, p.wait_ns)))
        return false;
      if (warp == 4 && lane == 0) TRACE(3, 16);
      tc_fence_after();
      for (int gl = 0; gl < GO; ++gl) {
        const int G = hc * NGC + rank * GO + gl;
        if (q_r.o_f32) {
          // float32 O: each lane stores its own head dim (a warp writes 128 contiguous bytes);
          // D2 is released only after the last column is stored
          float* of = static_cast<float*>(q_r.O) + u.o_row0 * rs + (int64_t)G * q_r.gq * D + d;
#pragma unroll
          for (int c32 = 0; c32 < NPV / 32; ++c32) {
            uint32_t o[32];
            if (have) {
              tmem_ld32(tl + 128u * gl + 32u * c32, o);
              tmem_wait_ld();
              reg_fence(o);
            } else {
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = 0u;
            }
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) {
              const int n = 32 * c32 + cc;
              const int c = n >> 3, pp = (n >> 2) & 1, h = n & 3;
              const int r = 8 * (c >> 2) + 4 * ((c >> 1) & 1) + 2 * pp + (c & 1);
              if (G < q_r.h_kv && h < q_r.gq && r >= ilo && r < ihi)
                of[(int64_t)r * rs + h * D] = __uint_as_float(o[cc]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_OEMPTY + gl));
          continue;
        }
        uint32_t pk[NPV / 2];  // columns (2u, 2u + 1) rounded to bf16
#pragma unroll
        for (int c32 = 0; c32 < NPV / 32; ++c32) {
          uint32_t o[32];
          if (have) {
            tmem_ld32(tl + 128u * gl + 32u * c32, o);
            tmem_wait_ld();
            reg_fence(o);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0u;
          }
#pragma unroll
          for (int u2 = 0; u2 < 16; ++u2)
            pk[16 * c32 + u2] = pack_bf2(__uint_as_float(o[2 * u2]), __uint_as_float(o[2 * u2 + 1]));
        }
        // D2 of this group is read: the next unit's P.V may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_OEMPTY + gl));
        if (G < q_r.h_kv) {
          const bool odd = lane & 1;
          __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(q_r.O) + u.o_row0 * rs +
                              (int64_t)G * q_r.gq * D + (d & ~1);
#pragma unroll
          for (int u2 = 0; u2 < NPV / 2; ++u2) {
            // columns n = 2 u2 (head h even) and n + 1 (head h + 1) of the same row
            const uint32_t mine = pk[u2];
            const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
            // even lane: column n at dims (d, d + 1); odd lane: column n + 1 at (d - 1, d)
            const uint32_t wv = odd ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
            const int n = 2 * u2 + (odd ? 1 : 0);
            const int c = n >> 3, pp = (n >> 2) & 1, h = n & 3;
            const int r = 8 * (c >> 2) + 4 * ((c >> 1) & 1) + 2 * pp + (c & 1);
            if (h < q_r.gq && r >= ilo && r < ihi)
              *reinterpret_cast<uint32_t*>(ob + (int64_t)r * rs + h * D) = wv;
          }
        }
      }
      if (warp == 4 && lane == 0) TRACE(3, 17);
      return true;
    };
    bool ok = true;
    int T = 0, K = 0;   // tiles converted, epilogues done
    int pk_unit = -1, pidx = 0;  // a unit whose epilogue is still to run (after the next unit's first tile)
    float amax = 0.0f;
    for (int idx = cl, ik = 0; idx < p.n_units && ok; idx += ncl, ++ik) {
      const Unit u = unit(ik, idx);
      if (!u.valid) continue;
      int kb = u.kb0;
      for (int t = 0; t < u.n_tiles && ok; ++t, ++T) {
        if (t == 1 && pk_unit >= 0) {
          ok = epilogue(pk_unit, pidx, K++);
          pk_unit = -1;
          if (!ok) break;
        }
        const int half = t % tpb;
        if (t > 0 && half == 0) kb = p.col_idx[u.rp0 + t / tpb];
        const bool kb_ok = kb >= 0 && kb <= u.qb;
        const int tok0 = kb * p.B + half * KT;
        const int ps = T % PSLOTS;
        // rows of this thread: window row 8 rank + 2m + rb, query position i_begin + that
        const int ibase = u.i_begin + rank * RM + rb;
        const bool full = kb_ok && tok0 + KT - 1 <= u.i_begin + rank * RM;
        uint32_t pkA[HV / 2], pkB[HV / 2];
        for (int pair = 0; pair < 2 && ok; ++pair) {
          if (warp == 4 && lane == 0) TRACE(3, 9 + pair);
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_D1FULL + pair), T & 1, abort_flag, p.status, p.wait_ns));
          if (!ok) break;
          if (warp == 4 && lane == 0) TRACE(3, 11 + pair);
          tc_fence_after();
#pragma unroll
          for (int mm = 0; mm < 2; ++mm) {
            const int m = 2 * pair + mm;
            uint32_t hi[32], lo[32];
            tmem_ld32(tl + 256u + 64u * (uint32_t)m, hi);
            tmem_ld32(tl + 256u + 64u * (uint32_t)m + 32u, lo);
            tmem_wait_ld();
            reg_fence(hi);
            reg_fence(lo);
            if (mm == 1) {  // both M tiles of the half are in registers: release D1
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(B_D1EMPTY + pair));
            }
            const float mk = (kb_ok && tok0 + j <= ibase + 2 * m) ? 1.0f : 0.0f;
            uint32_t* pk = mm == 0 ? pkA : pkB;
#pragma unroll
            for (int v = 0; v < HV; v += 2) {
              float x0 = __uint_as_float(hi[v]) + __uint_as_float(lo[v]);
              float x1 = __uint_as_float(hi[v + 1]) + __uint_as_float(lo[v + 1]);
              if (!full) { x0 *= mk; x1 *= mk; }
              amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
              pk[v / 2] = pack_h2(x0, x1);
            }
          }
          // the slot must have been consumed by all four owners (tile T - PSLOTS)
          if (pair == 0 && T >= PSLOTS) {
            ok = __all_sync(0xffffffffu, mbar_wait<true>(bar(B_PEMPTY + ps), ((T / PSLOTS) & 1) ^ 1,
                                                         abort_flag, p.status, p.wait_ns));
            if (!ok) break;
          }
          if (warp == 4 && lane == 0) TRACE(3, 13 + pair);
          // one 16-byte chunk per group: rows (2*(2 pair) + rb, 2*(2 pair + 1) + rb), 4 heads each
          const uint32_t c = 4u * (uint32_t)rank + 2u * (uint32_t)pair + (uint32_t)rb;
          const uint32_t off = OFF_P + (uint32_t)ps * PSLOT_BYTES + (c >> 3) * 8192u +
                               (uint32_t)j * 128u + (((c & 7u) ^ ((uint32_t)j & 7u)) << 4);
#pragma unroll
          for (int g = 0; g < NGC; ++g) {
            const int owner = g / GO, gl = g % GO;
            st_async16(rbase[owner] + off + (uint32_t)gl * PG_BYTES,
                       rbase[owner] + OFF_BAR + 8u * (uint32_t)(B_PFULL + ps),
                       pkA[2 * g], pkA[2 * g + 1], pkB[2 * g], pkB[2 * g + 1]);
          }
        }
        if (!ok) break;
      }
      if (!ok) break;
      if (pk_unit >= 0) {
        ok = epilogue(pk_unit, pidx, K++);
        pk_unit = -1;
        if (!ok) break;
      }
      pk_unit = ik;
      pidx = idx;
    }
    if (ok && pk_unit >= 0) ok = epilogue(pk_unit, pidx, K++);
    if (amax > F16_MAX) atomicOr(p.status, ST_RANGE);
    // every owner has consumed the slots this CTA filled last (their commits have arrived here)
    if (lane == 0)
      for (int k = 0; k < PSLOTS; ++k) {
        const int cnt = T > k ? (T - k - 1) / PSLOTS + 1 : 0;
        if (cnt) mbar_drain<true>(bar(B_PEMPTY + k), (cnt - 1) & 1);
      }
    __syncwarp();
  } else if (warp >= 8) {
    // ================================================================ V loaders
    // 128 threads; per tile 2 groups x 64 keys x 16 vectors of 8 dims: 16 vectors per thread.
    // A cursor runs one tile ahead: the loads of the next tile are in flight while this one is
    // converted and stored.
    const int tid = threadIdx.x - 8 * 32;
    bool ok = true;
    int T = 0;
    float amax = 0.0f;
    // cursor over this cluster's tiles in order (units without tiles are skipped)
    int c_ik = -1, c_idx = cl - ncl, c_t = 0, c_kb = -1;
    Unit c_u;
    c_u.n_tiles = 0;
    auto advance = [&]() -> bool {  // to the next tile; false when none is left
      ++c_t;
      while (c_t >= c_u.n_tiles) {
        ++c_ik;
        c_idx += ncl;
        if (c_idx >= p.n_units) return false;
        c_u = unit(c_ik, c_idx);
        if (!c_u.valid) c_u.n_tiles = 0;
        c_t = 0;
      }
      if (c_t % tpb == 0) c_kb = c_t == 0 ? c_u.kb0 : p.col_idx[c_u.rp0 + c_t / tpb];
      return true;
    };
    auto issue = [&](uint4 (&r)[16]) {
      const int half = c_t % tpb;
      const bool kb_ok = c_kb >= 0 && c_kb <= c_u.qb;
      if (!kb_ok && rank == 0 && tid == 0) atomicOr(p.status, ST_INDEX);
      const int tok0 = c_kb * p.B + half * KT;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int v = tid + 128 * i;
        const int gl = v >> 10, key = (v >> 4) & 63, ch = v & 15;
        const int G = hc * NGC + rank * GO + gl;
        const int tok = tok0 + key;
        r[i] = make_uint4(0u, 0u, 0u, 0u);
        if (kb_ok && tok < c_u.k_len && G < q_r.h_kv) {
          int64_t row = -1;
          if (!q_r.paged) {
            row = (int64_t)c_u.k0 + tok;
            if (row >= q_r.total_k) row = -1;
          } else {
            const int slot = tok / q_r.page_size;
            if (slot < q_r.max_pages) {
              const int pg = q_r.block_table[(int64_t)c_u.s * q_r.max_pages + slot];
              if (pg >= 0 && pg < q_r.n_pages) row = (int64_t)pg * q_r.page_size + tok % q_r.page_size;
              else atomicOr(p.status, ST_PAGE);
            }
          }
          if (row >= 0)
            r[i] = __ldg(reinterpret_cast<const uint4*>(q_r.V + (row * q_r.h_kv + G) * D + ch * 8));
        }
      }
    };
    uint4 ra[16], rb[16];
    bool have = advance();
    if (have) issue(ra);
    while (have && ok) {
      const bool more = advance();
      if (more) issue(rb);
      const int vs = T % VSLOTS;
      if (warp == 8 && lane == 0) TRACE(4, 18);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_VEMPTY + vs), ((T / VSLOTS) & 1) ^ 1, abort_flag,
                                             p.status, p.wait_ns));
      if (!ok) break;
      if (warp == 8 && lane == 0) TRACE(4, 19);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int v = tid + 128 * i;
        const int gl = v >> 10, key = (v >> 4) & 63, ch = v & 15;
        const uint32_t dst = sb + OFF_V + (uint32_t)vs * VSLOT_BYTES + (uint32_t)gl * VG_BYTES +
                             ((uint32_t)ch >> 3) * 8192u + (uint32_t)key * 128u +
                             ((((uint32_t)ch & 7u) ^ ((uint32_t)key & 7u)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                     "r"(bf2_to_h2(ra[i].x, amax)), "r"(bf2_to_h2(ra[i].y, amax)),
                     "r"(bf2_to_h2(ra[i].z, amax)), "r"(bf2_to_h2(ra[i].w, amax))
                     : "memory");
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_VFULL + vs));
      if (warp == 8 && lane == 0) TRACE(4, 20);
      ++T;
      have = more;
#pragma unroll
      for (int i = 0; i < 16; ++i) ra[i] = rb[i];
    }
    if (amax > F16_MAX) atomicOr(p.status, ST_RANGE);
  }
  tc_fence_before();
  __syncthreads();
  // no CTA leaves while a peer may still signal or write into it
  cluster_sync_all();
  if (*abort_flag) {  // stores a stopped peer issued may still be in flight towards this CTA
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < GRACE_NS) {}
  }
#ifdef MF_TRACE
  if (blockIdx.x < TRACE_CTAS)
    for (int e = threadIdx.x; e < TRACE_ROLES * TRACE_N; e += NT) {
      const int r = e / TRACE_N, k = e % TRACE_N;
      g_trace[blockIdx.x][r][k] = k == 0 ? (uint64_t)s_tn[r] : s_tr[r][k];
    }
#endif
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
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

bool encode(CUtensorMap* tm, const void* base, int rank, const uint64_t* dims,
            const uint64_t* strides_bytes, const uint32_t* box, std::string* err) {
  auto fn = get_encode();
  if (!fn) { *err = "cuTensorMapEncodeTiled unavailable"; return false; }
  uint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  dims, strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { *err = "cuTensorMapEncodeTiled failed: " + std::to_string((int)r); return false; }
  return true;
}

// clusters of four CTAs that can be resident at once on the current device (queried once per
// device: the answer depends on the GPC layout, not on the launch)
int max_clusters(std::string* err) {
  static std::mutex mu;
  static int cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> g(mu);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  cudaError_t e = cudaFuncSetAttribute(k_retrieve_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return 0; }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms / CS * CS), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, k_retrieve_tc, &cfg);
  if (e != cudaSuccess || n < 1) {
    *err = std::string("cudaOccupancyMaxActiveClusters: ") + cudaGetErrorString(e);
    return 0;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace

bool tc_supported(const mf_retrieve_desc& d) {
  if (d.flags & MF_RETRIEVE_FORCE_SIMT) return false;
  if (d.map_dtype != MF_BF16 || d.v_dtype != MF_BF16) return false;
  if (!(d.B == 64 || d.B == 128) || d.d != D) return false;
  if (d.h_kv <= 0 || d.h_r % d.h_kv != 0 || d.h_r / d.h_kv > GQP) return false;
  if (d.h_s <= 0 || d.h_s > 64) return false;
  if (d.paged && d.page_size < 1) return false;
  return true;
}

bool launch_retrieve_tc(const mf_retrieve_desc* const* ds, const RetrieveLayer* ls, int n,
                        uint32_t* status, cudaStream_t st, std::string* err) {
  if (n < 1 || n > NRMAX) { *err = "1 to 4 receivers per launch"; return false; }
  const mf_retrieve_desc& d0 = *ds[0];
  const RetrieveLayer& l0 = ls[0];
  const int B = d0.B;
  CUtensorMap tmA;
  {  // kept blocks [capacity][h_s][B][B]: dims (key j, sender head s, row i, block n)
    const uint64_t dims[4] = {(uint64_t)B, (uint64_t)d0.h_s, (uint64_t)B,
                              (uint64_t)std::max<int64_t>(l0.capacity, 1)};
    const uint64_t strides[3] = {(uint64_t)B * B * 2, (uint64_t)B * 2, (uint64_t)d0.h_s * B * B * 2};
    const uint32_t box[4] = {KT, SC, RM, 1};
    if (!encode(&tmA, l0.values, 4, dims, strides, box, err)) return false;
  }
  TcParams p{};
  p.row_ptr = l0.row_ptr; p.col_idx = l0.col_idx; p.capacity = l0.capacity;
  p.cu_q = d0.cu_seqlens_q; p.cu_k = d0.cu_seqlens_k; p.qblock_base = d0.qblock_base;
  p.nseq = d0.nseq;
  p.nqbq = (d0.max_seqlen_q + B - 1) / B + 1;  // a chunk may start inside a block
  p.wcs = B / WR;
  p.h_s = d0.h_s; p.nsc = (d0.h_s + SC - 1) / SC; p.B = B;
  p.nrecv = n;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  p.stall = wait_stall();
  int NH = 0;
  for (int k = 0; k < n; ++k) {
    const mf_retrieve_desc& d = *ds[k];
    const RetrieveLayer& l = ls[k];
    RecvParams& r = p.rv[k];
    r.W = l.W; r.O = l.O;
    r.o_f32 = (d.flags & MF_RETRIEVE_O_F32) ? 1 : 0;
    r.V = static_cast<const __nv_bfloat16*>(l.V);
    r.block_table = d.block_table; r.paged = d.paged; r.page_size = d.page_size;
    r.n_pages = d.n_pages; r.max_pages = d.max_pages; r.total_k = d.total_k;
    r.h_r = d.h_r; r.h_kv = d.h_kv; r.gq = d.h_r / d.h_kv;
    r.hcs = (d.h_kv + NGC - 1) / NGC;
    p.hh_base[k] = NH;
    NH += r.hcs;
  }
  p.hh_base[n] = NH;
  p.NH = NH;
  const int64_t n_units = (int64_t)p.nqbq * d0.nseq * p.wcs * NH;
  if (n_units == 0 || d0.max_seqlen_q == 0) return true;
  if (n_units >= ((int64_t)1 << 31)) { *err = "too many work units"; return false; }
  p.n_units = (int)n_units;
  const int mc = max_clusters(err);
  if (mc < 1) return false;
  // persistent clusters, a multiple of the head-chunk count (one receiver and one W^T each)
  int64_t ncl = std::min<int64_t>(n_units, mc);
  ncl = std::max<int64_t>(NH, ncl / NH * NH);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(ncl * CS), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_retrieve_tc, tmA, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  return true;
}

}  // namespace mfi

#ifdef MF_TRACE
extern "C" __attribute__((visibility("default"))) int mf_trace_dump(void* host, size_t bytes) {
  if (bytes < sizeof(mfi::g_trace)) return -1;
  if (cudaMemcpyFromSymbol(host, mfi::g_trace, sizeof(mfi::g_trace)) != cudaSuccess) return -2;
  static uint64_t zero[mfi::TRACE_CTAS][mfi::TRACE_ROLES][mfi::TRACE_N];
  if (cudaMemcpyToSymbol(mfi::g_trace, zero, sizeof(zero)) != cudaSuccess) return -3;
  return 0;
}
#endif
