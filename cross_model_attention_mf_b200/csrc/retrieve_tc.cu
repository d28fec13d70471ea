// Fused map retrieval on sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com),
// section "存不下、读得慢?三个工程优化手段", subsection 3 "算得省的:融合内核执行":
// read the kept sparse blocks, mix sender heads into receiver heads on chip,
// multiply by the receiver's V and accumulate, without materialising the
// receiver's dense map.  The pages' kernel is Triton on A800; this one is a
// new design for B200.
//
// Work item = (sequence, query block, 16-row chunk, 4 KV groups = 16 virtual
// receiver heads; a group of gq <= 4 heads is padded to 4).  The kernel is
// persistent: each CTA walks items blockIdx.x, blockIdx.x + gridDim.x, ... (the grid
// is a multiple of the head-chunk count, so a CTA keeps one head chunk and one W^T),
// and every ring runs across item boundaries, so the loads and the mixing of the
// next item overlap the tail of the current one.  For each kept 64-key tile:
//
//   mixing  D1[pos][(part, r)] = sum_s A_s[pos] * W_part[r][s]   tcgen05 M=128 N=32 K=16
//           pos = (row, key) of 2 rows x 64 keys (one M tile), A tile MN-major SW128
//           from TMA; B = W^T with W split into bf16 hi and lo parts stacked along N,
//           so one MMA per M tile and s-chunk keeps ~16 bits of W.  D1 holds the eight
//           32-column M tiles of one key tile in TMEM.
//   convert 16 warps read D1 (lane = position), form P = hi part + lo part (float32),
//           apply the causal mask and write P as P^T[key][(row, head)] (MN-major SW128)
//           per group: split into bf16 hi + lo (P = hi + lo to ~16 bits) for float32
//           O, on request, and in the first query block of a sequence (rows with at
//           most B keys, where |P| is largest); rounded once to bf16 elsewhere, as a
//           bf16 attention kernel rounds its P.
//   P.V     D2[dim][(row, head)] += V^T[dim][key] * P^T[key][(row, head)]
//           tcgen05 M=128 (d) N=64 K=16 per group, one MMA per K step and part of P;
//           V tile MN-major SW128 by TMA (contiguous or paged).  D2 stays in TMEM for
//           the whole row chunk.
// Every tcgen05.mma with N <= 64 occupies the tensor pipe about as long as any other
// (a fixed cost per instruction measured on B200), so the kernel's tensor time follows
// its MMA count: 16 mixing + 16 P.V MMAs per tile with P in one part, 32 P.V with two.
//
// Warp roles: 0 TMA producer of the map tiles; 1 mixing MMA issuer (+ TMEM owner);
// 2 P.V MMA issuer; 3 TMA producer of the V tiles (separate producers and issuers, so
// no stream waits behind another); 4-19 convert (four sets of four warps, one warp per
// TMEM lane quarter; set k converts the M tiles m = k, k + 4 for all 16 heads) and, once
// per item, run the O epilogue (set k reads D2 group k, releases it for the next item's
// P.V and stores O).  Barriers are tile- or half-tile-granular: a barrier operation costs
// hundreds of cycles.  Converters release D1 as soon as it is in registers, so the next
// tile's mixing overlaps the conversion; P^T and the V ring work in half tiles (groups
// 0-1, 2-3), so P.V of one half overlaps the conversion of the other.  Consumer warps
// wait with all 32 lanes (the hardware suspends such a warp; a lone polling lane would
// spin) and signal once per warp (lane 0 after __syncwarp).  TMEM: D2 in columns
// [0, 256), D1 in [256, 512).  Every mbarrier wait is bounded by a timer (mf_set_wait_limit,
// default 2 s): on expiry the CTA records ST_TIMEOUT, all roles stop, in-flight copies and
// MMAs are drained (bounded) and TMEM is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "mf_internal.cuh"

namespace mfi {
namespace {

constexpr int NT = 640;        // 20 warps
constexpr int CONV_SETS = 4;   // convert warp sets
constexpr int R = 16;          // query rows per CTA
constexpr int KT = 64;         // keys per tile
constexpr int NG = 4;          // KV groups per CTA
constexpr int GQP = 4;         // virtual heads per group
constexpr int HV = NG * GQP;   // virtual receiver heads per CTA
constexpr int D = 128;         // head dim
constexpr int SC = 16;         // sender heads per A chunk (one MMA K step)
constexpr int MT = R * KT / 128;  // M tiles (of 128 positions) per tile: 8
#ifndef MF_TC_A_STAGES
#define MF_TC_A_STAGES 2
#endif
constexpr int A_STAGES = MF_TC_A_STAGES;
// Half tiles (KV groups 2h, 2h + 1) flow through a ring of HS slots; a slot holds the half's
// V tiles (loaded by TMA) and its P^T (written by the converters), filled and freed together.
constexpr int PH = 2;   // groups per half tile
constexpr int HS = 2;   // half-tile slots: one key tile
constexpr uint32_t A_BYTES = R * SC * KT * 2;   // 32 KB
constexpr uint32_t VGRP_BYTES = KT * D * 2;     // 16 KB: one group's V tile
constexpr uint32_t V_BYTES = PH * VGRP_BYTES;   // 32 KB: V of one half tile
// A V slot holds the half tile's two groups as [page][d half][group][page rows][128 B]
// (contiguous V: one 64-row page), which is the order in which one TMA box over (64 dims, page
// rows, 2 kv heads, 2 d halves) lands, so a stage takes one copy per page; the P.V descriptors
// step through it per K step of 16 keys.
constexpr uint32_t PT_BYTES = KT * 64 * 2;      // 8 KB: one group's P^T (hi or lo)
constexpr uint32_t PSLOT_BYTES = 2 * PT_BYTES;  // hi + lo of one group
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_V = OFF_A + A_STAGES * A_BYTES;
constexpr uint32_t OFF_P = OFF_V + HS * V_BYTES;
constexpr uint32_t PHALF_BYTES = PH * PSLOT_BYTES;  // 32 KB
constexpr uint32_t OFF_W = OFF_P + HS * PHALF_BYTES;
constexpr uint32_t W_CHUNK = 1024;              // W^T (32 rows = hi, lo) per s-chunk
constexpr uint32_t W_BYTES_MAX = 4 * W_CHUNK;   // up to 4 chunks (h_s <= 64)
constexpr int ITEMS_MAX = 64;                     // work items per CTA decoded up front
constexpr uint32_t ITEM_BYTES = 64;
constexpr uint32_t OFF_ITEMS = OFF_W + W_BYTES_MAX;
constexpr uint32_t OFF_BAR = OFF_ITEMS + ITEMS_MAX * ITEM_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory of one CTA");

// barrier slots (8 bytes each)
enum {
  B_AFULL = 0, B_AEMPTY = B_AFULL + A_STAGES, B_HFULL = B_AEMPTY + A_STAGES,
  B_HEMPTY = B_HFULL + HS, B_D1FULL = B_HEMPTY + HS, B_D1EMPTY = B_D1FULL + 1,
  B_OFULL = B_D1EMPTY + 1,
  B_OEMPTY = B_OFULL + 1, B_DRAIN1 = B_OEMPTY + 2, B_DRAIN2 = B_DRAIN1 + 1,
  B_NEVER = B_DRAIN2 + 1,  // test stall: nothing ever arrives here
  B_COUNT = B_NEVER + 1
};
static_assert(B_COUNT * 8 <= 512, "barrier area");

// instruction descriptors (kind::f16): D f32, A/B bf16, majors, N >> 3, M >> 4
constexpr uint32_t IDESC_MIX = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (0u << 16) |
                               ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                              ((64u >> 3) << 17) | ((128u >> 4) << 24);

constexpr int NRMAX = 4;  // receivers served by one launch (one BSR, several W / V / O)

// one receiver: its head map, V and O (and its V paging)
struct RecvParams {
  const float* W;  // [h_r][h_s]
  void* O;         // bf16, or float32 when o_f32
  int o_f32;
  int p_split;     // P in hi and lo parts in every item
  const int32_t* block_table;
  int paged, page_size, n_pages, max_pages;
  int total_k;     // V rows (contiguous V): the out-of-range row that reads zeros
  int h_r, h_kv, gq, hcs;
};
struct TcParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  int64_t capacity;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* qblock_base;
  int nqbq, rcs;    // query blocks, row chunks per block
  int NH;           // head chunks of all receivers together
  int hh_base[NRMAX + 1];  // first head chunk of each receiver
  int nrecv;
  int n_items;
  int h_s, nsc, B;
  RecvParams rv[NRMAX];
  uint32_t* status;
  uint64_t wait_ns;  // limit of every pipeline wait
  int stall;         // test: the mixing issuer first waits on B_NEVER
  int dep_wait;      // the call's first launch: wait for the previous kernel on the stream
};
struct VMaps {
  CUtensorMap m[NRMAX];
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
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
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
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint64_t limit_ns) {
  if (mbar_try(bar, parity)) return true;
  uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
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
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* tm, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
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
// (above the tcgen05.wait::ld that makes v valid, or above a barrier signal that should go
// out before the arithmetic on v).
__device__ __forceinline__ void reg_fence(uint32_t (&v)[32]) {
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),
                 "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),
                 "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
                 "+r"(v[30]), "+r"(v[31]));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Optional timeline trace (compile with -DMF_TRACE): per CTA and role, SM-clock stamps of
// pipeline events kept in shared memory and copied out at the end, read back with
// mf_trace_dump().  Each role has a single writing thread.
#ifdef MF_TRACE
constexpr int TRACE_CTAS = 160, TRACE_N = 256, TRACE_ROLES = 6;
__device__ uint64_t g_trace[TRACE_CTAS][TRACE_ROLES][TRACE_N];
#define TRACE(role, code)                                                            \
  do {                                                                               \
    const int n_ = s_tn[role];                                                       \
    if (n_ < TRACE_N - 1) {                                                          \
      s_tr[role][1 + n_] = ((uint64_t)(code) << 56) | ((uint64_t)clock64() & ((1ull << 56) - 1)); \
      s_tn[role] = n_ + 1;                                                           \
    }                                                                                \
  } while (0)
#else
#define TRACE(role, code)
#endif

// ------------------------------------------------------------------ kernel
struct Item {
  int s, qb, q0, i_begin, row_lo, row_hi, k_len, n_tiles;
  int k0;   // first key row of the sequence (cu_seqlens_k[s])
  int kb0;  // key block of the row's first kept block (col_idx[rp0]), -1 without tiles
  int64_t rp0;
  int64_t o_row0;  // O row of query position i_begin (cu_seqlens_q[s] + i_begin - q0)
  bool valid, bsr_ok;
};
static_assert(sizeof(Item) <= ITEM_BYTES, "item table slot");

// item idx = ((s * nqbq + qbl) * rcs + rc) * NH + hh, hh = a receiver's head chunk;
// identical in every role
__device__ __forceinline__ Item decode(const TcParams& p, int idx) {
  Item it;
  it.valid = false;
  it.bsr_ok = true;
  it.n_tiles = 0;
  idx /= p.NH;
  const int rc = idx % p.rcs;
  idx /= p.rcs;
  const int qbl = idx % p.nqbq;
  const int s = idx / p.nqbq;
  const int q_len = p.cu_q[s + 1] - p.cu_q[s];
  const int k_len = p.cu_k[s + 1] - p.cu_k[s];
  const int q0 = k_len - q_len;
  if (q_len <= 0 || q0 < 0) return it;
  const int qb = q0 / p.B + qbl;
  if ((int64_t)qb * p.B >= k_len) return it;
  const int i_begin = qb * p.B + rc * R;
  const int row_lo = max(q0, i_begin), row_hi = min(k_len, i_begin + R);
  if (row_lo >= row_hi) return it;
  const int64_t brow = (int64_t)p.qblock_base[s] + qb;
  const int64_t rp0 = p.row_ptr[brow], rp1 = p.row_ptr[brow + 1];
  it.bsr_ok = rp0 >= 0 && rp1 >= rp0 && rp1 <= p.capacity && rp1 - rp0 <= qb + 1;
  it.n_tiles = it.bsr_ok ? (int)(rp1 - rp0) * (p.B / KT) : 0;
  it.s = s; it.qb = qb; it.q0 = q0; it.i_begin = i_begin; it.row_lo = row_lo;
  it.row_hi = row_hi; it.k_len = k_len; it.rp0 = rp0; it.k0 = p.cu_k[s];
  it.kb0 = it.n_tiles > 0 ? p.col_idx[rp0] : -1;
  it.o_row0 = (int64_t)p.cu_q[s] + (i_begin - q0);
  it.valid = true;
  return it;
}

__global__ void __launch_bounds__(NT, 1)
    k_retrieve_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ VMaps tmVs,
                  const __grid_constant__ TcParams p) {
  // Every launch is a programmatic dependent launch.  A later launch of the same call reads
  // nothing this grid writes, so it may take SMs as soon as this grid's CTAs exit; the call's
  // first launch waits for the previous kernel on the stream (below, before its first global
  // access) and only then lets the later launches start.
  if (!p.dep_wait) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
  // receiver and head chunk: constant per CTA (gridDim.x is a multiple of NH)
  const int hh = blockIdx.x % p.NH;
  int ri = 0;
  while (ri + 1 < p.nrecv && hh >= p.hh_base[ri + 1]) ++ri;
  const RecvParams& q_r = p.rv[ri];
  const CUtensorMap* tmV = &tmVs.m[ri];
  const int hc = hh - p.hh_base[ri];
  const int tpb = p.B / KT;
  // P.V multiplies P in bf16 hi and lo parts (P to ~16 bits) for float32 O, when the caller asks
  // for it, and in the first query block of a sequence, whose rows see at most B keys and carry
  // the largest |P|; elsewhere P is rounded once to bf16, as in a bf16 attention kernel
  const bool split_all = q_r.o_f32 != 0 || q_r.p_split != 0;
  auto split_p = [&](const Item& q) { return split_all || q.qb == 0; };

  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + OFF_BAR;
  auto bar = [&](int k) { return bar0 + 8u * (uint32_t)k; };
  // item k of this CTA (idx = blockIdx.x + k * gridDim.x): the first ITEMS_MAX come from the
  // table decoded once below, later ones are decoded where they are needed
  Item* s_items = reinterpret_cast<Item*>(smem + OFF_ITEMS);
  auto item = [&](int k, int idx) -> Item { return k < ITEMS_MAX ? s_items[k] : decode(p, idx); };

  // ---- setup
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int k = 0; k < A_STAGES; ++k) { mbar_init(bar(B_AFULL + k), 1); mbar_init(bar(B_AEMPTY + k), 1); }
    for (int k = 0; k < HS; ++k) {
      mbar_init(bar(B_HFULL + k), 1 + 4 * CONV_SETS);  // V producer + converter warps
      mbar_init(bar(B_HEMPTY + k), 1);
    }
    mbar_init(bar(B_D1FULL), 1);
    mbar_init(bar(B_D1EMPTY), 4 * CONV_SETS);
    for (int h = 0; h < NG / PH; ++h) mbar_init(bar(B_OEMPTY + h), 4 * PH);  // epilogue warps
    mbar_init(bar(B_OFULL), 1);
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
  if (p.dep_wait) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  // W^T of this CTA's 16 virtual heads, bf16, K-major without swizzle, 32 rows per s:
  // row n < 16 is the hi part of head n, row 16 + n its lo part.  Element (n, s) at
  // (s/8)*512 + (n/8)*128 + (n%8)*16 + (s%8)*2.
  {
    const int ks = p.nsc * SC;
    uint16_t* wt = reinterpret_cast<uint16_t*>(smem + OFF_W);
    for (int e = threadIdx.x; e < HV * ks; e += NT) {
      const int rv = e / ks, hs = e % ks;
      const int G = hc * NG + rv / GQP, q = rv % GQP;
      float w = 0.0f;
      if (q < q_r.gq && G < q_r.h_kv && hs < p.h_s) w = q_r.W[(int64_t)(G * q_r.gq + q) * p.h_s + hs];
      __nv_bfloat16 hi = __float2bfloat16_rn(w);
      __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
      const int base = (hs >> 3) * 512 + (hs & 7) * 2;
      wt[(base + (rv >> 3) * 128 + (rv & 7) * 16) >> 1] = *reinterpret_cast<uint16_t*>(&hi);
      wt[(base + ((rv + 16) >> 3) * 128 + (rv & 7) * 16) >> 1] = *reinterpret_cast<uint16_t*>(&lo);
    }
  }
  // the item table: one decode per item instead of one per item and role; decoded by the last
  // ITEMS_MAX threads (no W^T work while h_s <= 32), so its chain of loads overlaps W^T's
  if (threadIdx.x >= NT - ITEMS_MAX) {
    const int k = threadIdx.x - (NT - ITEMS_MAX);
    const int idx = blockIdx.x + k * gridDim.x;
    if (idx < p.n_items) s_items[k] = decode(p, idx);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0 || warp == 3) {
    // ================================================================ TMA producers
    // warp 0: map tiles (A chunks) in mixing order; warp 3: V tiles in P.V order (one stage
    // per half tile = groups 2h, 2h + 1)
    if (lane == 0) {
      const bool is_a = warp == 0;
      int as = 0, vs = 0;
      uint32_t aph = 0, vph = 0;
      int a_issued = 0, v_issued = 0;
      bool ok = true;
      for (int idx = blockIdx.x, ik = 0; idx < p.n_items && ok; idx += gridDim.x, ++ik) {
        const Item it = item(ik, idx);
        if (!it.valid) continue;
        if (is_a) TRACE(0, 1);
        if (is_a && !it.bsr_ok) atomicOr(p.status, ST_INDEX);
        const int rc = (idx / p.NH) % p.rcs;
        // key block of the current kept block and, loaded one block ahead, of the next one
        const int nblk = it.n_tiles / tpb;
        int kb_cur = it.kb0, kb_nxt = (!is_a && nblk > 1) ? p.col_idx[it.rp0 + 1] : -1;
        for (int t = 0; t < it.n_tiles && ok; ++t) {
          const int64_t e = it.rp0 + t / tpb;
          const int half = t % tpb;
          if (!is_a && t > 0 && half == 0) {
            kb_cur = kb_nxt;
            if (t / tpb + 1 < nblk) kb_nxt = p.col_idx[e + 1];
          }
          if (is_a) {
            for (int c = 0; c < p.nsc && ok; ++c) {
              if (!(ok = mbar_wait(bar(B_AEMPTY + as), aph ^ 1, abort_flag, p.status, p.wait_ns))) break;
              TRACE(0, 3);
              mbar_expect_tx(bar(B_AFULL + as), A_BYTES);
              tma_load_4d(sb + OFF_A + as * A_BYTES, &tmA, bar(B_AFULL + as), half * KT, c * SC,
                          rc * R, (int)e);
              TRACE(0, 2);
              ++a_issued;
              if (++as == A_STAGES) { as = 0; aph ^= 1; }
            }
            continue;
          }
          const int kb = kb_cur;
          const bool kb_ok = kb >= 0 && kb <= it.qb;
          if (!kb_ok) atomicOr(p.status, ST_INDEX);
          const int tok0 = kb * p.B + half * KT;
          if (!q_r.paged) {
            const int row = kb_ok ? it.k0 + tok0 : q_r.total_k;  // out of range reads 0
            for (int h = 0; h < NG / PH && ok; ++h) {
              if (!(ok = mbar_wait(bar(B_HEMPTY + vs), vph ^ 1, abort_flag, p.status, p.wait_ns))) break;
              TRACE(5, 4);
              mbar_expect_tx(bar(B_HFULL + vs), V_BYTES);
              // one copy: 64 keys of both groups and both d halves (coordinates: dim, token,
              // kv head, d half; a head past h_kv reads zeros)
              tma_load_4d(sb + OFF_V + vs * V_BYTES, tmV, bar(B_HFULL + vs), 0, row,
                          hc * NG + h * PH, 0);
              ++v_issued;
              TRACE(5, 3);
              if (++vs == HS) { vs = 0; vph ^= 1; }
            }
            continue;
          }
          // paged V: the tile's page ids, looked up once for all groups (independent loads)
          const int ps = q_r.page_size;
          int pages[KT / 8];
          uint32_t looked = 0;  // bit q: page q's id comes from the block table
#pragma unroll
          for (int q = 0; q < KT / 8; ++q) {
            const int tok = tok0 + q * ps, slot = tok / ps;
            pages[q] = q_r.n_pages;  // out of range: the copy reads zeros
            if (q * ps < KT && kb_ok && tok < it.k_len && slot < q_r.max_pages) {
              pages[q] = q_r.block_table[(int64_t)it.s * q_r.max_pages + slot];
              looked |= 1u << q;
            }
          }
          for (int h = 0; h < NG / PH && ok; ++h) {
            if (!(ok = mbar_wait(bar(B_HEMPTY + vs), vph ^ 1, abort_flag, p.status, p.wait_ns))) break;
            TRACE(5, 4);
            if (h == 0) {
              // checked after the first wait, so that the lookups' latency overlaps it
#pragma unroll
              for (int q = 0; q < KT / 8; ++q)
                if (((looked >> q) & 1u) && (pages[q] < 0 || pages[q] >= q_r.n_pages)) {
                  atomicOr(p.status, ST_PAGE);
                  pages[q] = q_r.n_pages;
                }
            }
            mbar_expect_tx(bar(B_HFULL + vs), V_BYTES);
            // one copy per page: its rows of both groups and both d halves (coordinates: dim,
            // row in page, kv head, d half, page)
            const uint32_t dst = sb + OFF_V + vs * V_BYTES;
            const int G = hc * NG + h * PH;
#pragma unroll
            for (int q = 0; q < KT / 8; ++q) {
              if (q * ps >= KT) break;
              tma_load_5d(dst + (uint32_t)(q * 4 * ps * 128), tmV, bar(B_HFULL + vs), 0, 0, G, 0,
                          pages[q]);
            }
            ++v_issued;
            TRACE(5, 3);
            if (++vs == HS) { vs = 0; vph ^= 1; }
          }
        }
      }
      // drain: wait (bounded) for the last copy issued into every stage
      for (int k = 0; k < A_STAGES; ++k) {
        const int cnt = a_issued > k ? (a_issued - k - 1) / A_STAGES + 1 : 0;
        if (cnt) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try(bar(B_AFULL + k), (cnt - 1) & 1) && globaltimer() - t0 < DRAIN_NS) {}
        }
      }
      // (a V slot's phase also needs the converters' arrivals: after an abort this wait runs
      // out its bounded time)
      for (int k = 0; k < HS; ++k) {
        const int cnt = v_issued > k ? (v_issued - k - 1) / HS + 1 : 0;
        if (cnt) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try(bar(B_HFULL + k), (cnt - 1) & 1) && globaltimer() - t0 < DRAIN_NS) {}
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ mixing MMA issuer
    if (lane == 0) {
      int as = 0;
      uint32_t aph = 0;
      bool ok = true;
      int T = 0;  // tiles processed so far
      const uint64_t wdesc0 = smem_desc(sb + OFF_W, 512u, 128u, 0u);
      const uint64_t adesc0 = smem_desc(sb + OFF_A, 2048u, 1024u, 2u);
      // test stall: a wait that can only run out (the whole CTA then stops as on any timeout)
      if (p.stall) ok = mbar_wait(bar(B_NEVER), 0, abort_flag, p.status, p.wait_ns);
      for (int idx = blockIdx.x, ik = 0; idx < p.n_items && ok; idx += gridDim.x, ++ik) {
        const Item it = item(ik, idx);
        if (!it.valid) continue;
        TRACE(1, 1);
        for (int t = 0; t < it.n_tiles && ok; ++t, ++T) {
          // D1 must have been read out by the previous tile's converters
          if (!(ok = mbar_wait(bar(B_D1EMPTY), (T & 1) ^ 1, abort_flag, p.status, p.wait_ns))) break;
          tc_fence_after();
          // chunk-major: each s-chunk is mixed into all eight M tiles, then its stage is freed
          for (int c = 0; c < p.nsc && ok; ++c) {
            if (!(ok = mbar_wait(bar(B_AFULL + as), aph, abort_flag, p.status, p.wait_ns))) break;
            tc_fence_after();
            if (c == 0) TRACE(1, 3);
            const uint64_t ad = adesc0 + (((uint32_t)as * A_BYTES) >> 4);
            const uint64_t wd = wdesc0 + ((c * W_CHUNK) >> 4);
#pragma unroll
            for (int m = 0; m < MT; ++m)
              tc_mma(tmem + 256u + 32u * (uint32_t)m, ad + ((m * 4096u) >> 4), wd, IDESC_MIX,
                     c > 0 ? 1u : 0u);
            TRACE(1, 5);
            tc_commit(bar(B_AEMPTY + as));
            if (++as == A_STAGES) { as = 0; aph ^= 1; }
          }
          if (!ok) break;
          tc_commit(bar(B_D1FULL));
          TRACE(1, 4);
        }
      }
      tc_commit(bar(B_DRAIN1));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(B_DRAIN1), 0) && globaltimer() - t0 < DRAIN_NS) {}
    }
  } else if (warp == 2) {
    // ================================================================ P.V MMA issuer
    if (lane == 0) {
      int vs = 0;
      uint32_t vph = 0;
      bool ok = true;
      int T = 0, K = 0;  // tiles and items processed so far
      // V^T operand: the two d halves of a page 2 x page rows x 128 bytes apart; 8-key groups
      // 1024 bytes apart, or with 8-token pages the next page (2 d halves x 2 groups x 8 rows x
      // 128 bytes further)
      const int vps = q_r.paged ? q_r.page_size : KT;  // rows per V page in the slot
      const uint64_t vdesc0 =
          smem_desc(sb + OFF_V, (uint32_t)(2 * vps * 128), vps == 8 ? 4096u : 1024u, 2u);
      // offset (16-byte units) of group gl's keys [16 k, 16 k + 16) within a d half of the slot:
      // vbase[k] + gl * vgrp, worked out once (the issuing thread sets the MMA rate)
      uint32_t vbase[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = (16 * k) / vps, r0 = (16 * k) % vps;
        vbase[k] = (uint32_t)(q * (4 * vps * 128) + r0 * 128) >> 4;
      }
      const uint32_t vgrp = (uint32_t)(vps * 128) >> 4;
      const uint64_t pdesc0 = smem_desc(sb + OFF_P, 8192u, 1024u, 2u);
      for (int idx = blockIdx.x, ik = 0; idx < p.n_items && ok; idx += gridDim.x, ++ik) {
        const Item it = item(ik, idx);
        if (!it.valid) continue;
        TRACE(4, 6);
        for (int t = 0; t < it.n_tiles && ok; ++t, ++T) {
          for (int h = 0; h < NG / PH && ok; ++h) {
            // the half's V tiles and P^T are in slot vs
            if (!(ok = mbar_wait(bar(B_HFULL + vs), vph, abort_flag, p.status, p.wait_ns))) break;
            TRACE(4, 8);
            // the previous item's epilogue must have read this half of D2 out
            if (t == 0 && K > 0) {
              if (!(ok = mbar_wait(bar(B_OEMPTY + h), (K - 1) & 1, abort_flag, p.status, p.wait_ns))) break;
              TRACE(4, 9);
            }
            tc_fence_after();
            TRACE(4, 5);
            // the MMAs of the half's two groups are interleaved, so consecutive MMAs accumulate
            // into different D2 columns
            const uint64_t pd = pdesc0 + ((vs * PHALF_BYTES) >> 4);
            const uint64_t vd = vdesc0 + ((vs * V_BYTES) >> 4);
            // P in its hi and lo parts, or rounded to bf16 (the item's split rule)
            // (contiguous V: the offsets are constants)
            auto issue = [&](auto parts, auto contiguous) {
              constexpr int NP = decltype(parts)::value;
#pragma unroll
              for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int part = 0; part < NP; ++part)
#pragma unroll
                  for (int gl = 0; gl < PH; ++gl)
                    tc_mma(tmem + 64u * (uint32_t)(h * PH + gl),
                           vd + (decltype(contiguous)::value
                                     ? (uint32_t)((gl * KT * 128 + k * 16 * 128) >> 4)
                                     : vbase[k] + (uint32_t)gl * vgrp),
                           pd + ((gl * PSLOT_BYTES + part * PT_BYTES + k * 2048u) >> 4), IDESC_PV,
                           (t > 0 || k > 0 || part > 0) ? 1u : 0u);
            };
            const bool split = split_p(it);
            if (!q_r.paged) {
              if (split) issue(std::integral_constant<int, 2>{}, std::true_type{});
              else issue(std::integral_constant<int, 1>{}, std::true_type{});
            } else {
              if (split) issue(std::integral_constant<int, 2>{}, std::false_type{});
              else issue(std::integral_constant<int, 1>{}, std::false_type{});
            }
            TRACE(4, 10);
            tc_commit(bar(B_HEMPTY + vs));  // V and P^T of the slot consumed
            if (++vs == HS) { vs = 0; vph ^= 1; }
          }
        }
        if (!ok) break;
        if (it.n_tiles == 0 && K > 0) {  // take the epilogue's phases in order all the same
          for (int h = 0; h < NG / PH && ok; ++h)
            ok = mbar_wait(bar(B_OEMPTY + h), (K - 1) & 1, abort_flag, p.status, p.wait_ns);
          if (!ok) break;
        }
        tc_commit(bar(B_OFULL));  // D2 of this item complete (immediate when it has no tile)
        TRACE(4, 7);
        ++K;
      }
      tc_commit(bar(B_DRAIN2));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(B_DRAIN2), 0) && globaltimer() - t0 < DRAIN_NS) {}
    }
  } else if (warp < 4 + 4 * CONV_SETS) {
    // ================================================================ convert P (hi + lo)
    // Warp (set, quarter) owns TMEM lanes of its quarter in M tiles set and set + 4, i.e.
    // key j of rows 2 set + rb and 2 set + 8 + rb, which is exactly one 16-byte chunk of the
    // P^T row of key j (D2 column n = 8 (2 set + rb) + 4 mi + head): one conflict-free
    // 16-byte store per group for the hi part and one for the lo part.
    const int quarter = warp & 3;
    const int set = (warp - 4) >> 2;
    const int lrow = quarter * 32 + lane;  // TMEM lane = position in an M tile
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const int j = lrow & 63, rb = lrow >> 6;
    const uint32_t choff =
        (uint32_t)j * 128u + ((((uint32_t)(2 * set + rb)) ^ ((uint32_t)j & 7u)) << 4);
    // O epilogue of an item, shared by the 16 warps: warp (set, quarter) reads D2 group g = set
    // (64 columns) for head dims [32 quarter, 32 quarter + 32), releases it and stores O
    const int ng = min(NG, q_r.h_kv - hc * NG);  // real groups of this head chunk
    const int64_t rs = (int64_t)q_r.h_r * D;     // O row stride
    // the item (table slot ek, index eidx) is re-read from the item table here
    auto epilogue = [&](int ek, int eidx, int K) -> bool {
      const Item q = item(ek, eidx);
      const bool have = q.n_tiles > 0;
      const int ilo = q.row_lo - q.i_begin, ihi = q.row_hi - q.i_begin;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), K & 1, abort_flag, p.status, p.wait_ns)))
        return false;
      tc_fence_after();
      if (warp == 4 && lane == 0) TRACE(3, 1);
      const int g = set;
      if (q_r.o_f32) {
        // float32 O: each lane stores its own head dim (a warp writes 128 contiguous bytes);
        // D2 is released once every column is stored
        float* of = static_cast<float*>(q_r.O) +
                    (q.o_row0 * q_r.h_r + (int64_t)(hc * NG + g) * q_r.gq) * D + quarter * 32 + lane;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t o[32];
          if (have) {
            tmem_ld32(tl + 64u * g + 32u * hh, o);
            tmem_wait_ld();
            reg_fence(o);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = 0u;
          }
          // column n = 8 c + 4 mi + head holds row 2 (c / 2) + 8 mi + c % 2
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            const int n = 32 * hh + cc, c8 = n >> 3;
            const int ii = 2 * (c8 >> 1) + 8 * ((n >> 2) & 1) + (c8 & 1), rv = n & 3;
            if (g < ng && rv < q_r.gq && ii >= ilo && ii < ihi) of[ii * rs + rv * D] = __uint_as_float(o[cc]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_OEMPTY + g / PH));
        return true;
      }
      uint32_t pr[32];  // the group's 64 columns rounded to bf16, as pairs (2u, 2u + 1)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[32];
        if (have) {
          tmem_ld32(tl + 64u * g + 32u * hh, o);
          tmem_wait_ld();
          reg_fence(o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u)
          pr[16 * hh + u] = pack_bf16(__uint_as_float(o[2 * u]), __uint_as_float(o[2 * u + 1]));
      }
      // D2 of this group is read: the next item's P.V may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_OEMPTY + g / PH));
      if (warp == 4 && lane == 0) TRACE(3, 2);
      if (g < ng) {
        __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(q_r.O) +
                            (q.o_row0 * q_r.h_r + (int64_t)(hc * NG + g) * q_r.gq) * D + quarter * 32 + lane;
        // column n = 8 c + 4 mi + head holds row 2 (c / 2) + 8 mi + c % 2
#pragma unroll
        for (int u = 0; u < 32; ++u) {
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int n = 2 * u + b, c8 = n >> 3;
            const int ii = 2 * (c8 >> 1) + 8 * ((n >> 2) & 1) + (c8 & 1), rv = n & 3;
            if (rv < q_r.gq && ii >= ilo && ii < ihi)
              *reinterpret_cast<uint16_t*>(ob + ii * rs + rv * D) =
                  (uint16_t)(b ? pr[u] >> 16 : pr[u] & 0xFFFFu);
          }
        }
      }
      return true;
    };
    bool ok = true;
    int T = 0, K = 0;     // tiles converted, epilogues done
    // an item whose O epilogue is still to run (pk < 0: none): it runs after the next item's
    // first tile is converted, so P.V never waits for the stores
    int pk = -1, pidx = 0;
    int kb_prev = -1;  // key block of the previous tile (tiles of one kept block share it)
    for (int idx = blockIdx.x, ik = 0; idx < p.n_items && ok; idx += gridDim.x, ++ik) {
      const Item it = item(ik, idx);
      if (!it.valid) continue;
      for (int t = 0; t < it.n_tiles && ok; ++t, ++T) {
        // the previous item's epilogue, after this item's first tile
        if (t == 1 && pk >= 0) {
          ok = epilogue(pk, pidx, K++);
          pk = -1;
          if (!ok) break;
        }
        const int64_t e = it.rp0 + t / tpb;
        const int half = t % tpb;
        const int kb = half == 0 && t == 0 ? it.kb0 : (half == 0 ? p.col_idx[e] : kb_prev);
        kb_prev = kb;
        const bool kb_ok = kb >= 0 && kb <= it.qb;
        const int tok0 = kb * p.B + half * KT;
        // warp-uniform control flow: tcgen05.ld is a warp-collective instruction
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_D1FULL), T & 1, abort_flag, p.status, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
        if (warp == 4 && lane == 0) TRACE(2, 1);
        // both M tiles into registers first, so that D1 is released as early as possible
        // (columns 0-15: A.W_hi of the 16 heads, 16-31: A.W_lo)
        uint32_t v[MT / CONV_SETS][32];
#pragma unroll
        for (int mi = 0; mi < MT / CONV_SETS; ++mi)
          tmem_ld32(tl + 256u + 32u * (uint32_t)(set + mi * CONV_SETS), v[mi]);
        tmem_wait_ld();
        if (warp == 4 && lane == 0) TRACE(2, 5);
        // D1 is in registers: the next tile's mixing may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_D1EMPTY));
#pragma unroll
        for (int mi = 0; mi < MT / CONV_SETS; ++mi) reg_fence(v[mi]);
        // Split items: P = hi + lo with hi = P truncated to bf16 and lo = bf16(P - hi), both
        // written.  Other items: P rounded to bf16, one part.  Both variants are written out, so
        // that neither carries the other's registers.  A tile wholly below the diagonal of every
        // row needs no causal mask.
        auto convert = [&](auto lo_parts) -> bool {
          constexpr bool SPLIT = decltype(lo_parts)::value;
          const bool full = kb_ok && tok0 + KT - 1 <= it.i_begin;
          // per group: the chunk's packed hi (or only) words and lo words
          uint32_t hw[NG][4], lw[SPLIT ? NG : 1][4];
#pragma unroll
          for (int mi = 0; mi < MT / CONV_SETS; ++mi) {
            const int ii = 2 * (set + mi * CONV_SETS) + rb;
            const float mk = kb_ok && tok0 + j <= it.i_begin + ii ? 1.0f : 0.0f;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
#pragma unroll
              for (int c = 0; c < 4; c += 2) {
                float x0 =
                    __uint_as_float(v[mi][4 * g + c]) + __uint_as_float(v[mi][16 + 4 * g + c]);
                float x1 = __uint_as_float(v[mi][4 * g + c + 1]) +
                           __uint_as_float(v[mi][16 + 4 * g + c + 1]);
                if (!full) {
                  x0 *= mk;
                  x1 *= mk;
                }
                if constexpr (SPLIT) {
                  const uint32_t b0 = __float_as_uint(x0) & 0xFFFF0000u;
                  const uint32_t b1 = __float_as_uint(x1) & 0xFFFF0000u;
                  hw[g][2 * mi + c / 2] = __byte_perm(b0, b1, 0x7632);
                  // P - hi is exact in f32; one rounding to bf16 for the pair
                  lw[SPLIT ? g : 0][2 * mi + c / 2] =
                      pack_bf16(x0 - __uint_as_float(b0), x1 - __uint_as_float(b1));
                } else {
                  hw[g][2 * mi + c / 2] = pack_bf16(x0, x1);
                }
              }
            }
          }
          if (warp == 4 && lane == 0) TRACE(2, 3);
          bool ok_ = true;
#pragma unroll
          for (int h = 0; h < NG / PH; ++h) {
            // this half of the P buffer must have been consumed by the previous tile's P.V
            const int hq = T * (NG / PH) + h, ps = hq % HS;  // half-tile count, slot
            ok_ = __all_sync(0xffffffffu, mbar_wait(bar(B_HEMPTY + ps), ((hq / HS) & 1) ^ 1,
                                                    abort_flag, p.status, p.wait_ns));
            if (!ok_) break;
            if (warp == 4 && lane == 0) TRACE(2, 4);
#pragma unroll
            for (int gl = 0; gl < PH; ++gl) {
              const int g = h * PH + gl;
              const uint32_t pt = sb + OFF_P + ps * PHALF_BYTES + gl * PSLOT_BYTES + choff;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pt), "r"(hw[g][0]),
                           "r"(hw[g][1]), "r"(hw[g][2]), "r"(hw[g][3])
                           : "memory");
              if constexpr (SPLIT)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pt + PT_BYTES),
                             "r"(lw[SPLIT ? g : 0][0]), "r"(lw[SPLIT ? g : 0][1]),
                             "r"(lw[SPLIT ? g : 0][2]), "r"(lw[SPLIT ? g : 0][3])
                             : "memory");
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_HFULL + ps));
          }
          return ok_;
        };
        ok = split_p(it) ? convert(std::true_type{}) : convert(std::false_type{});
        if (!ok) break;
        if (warp == 4 && lane == 0) TRACE(2, 2);
      }
      if (!ok) break;
      if (pk >= 0) {
        ok = epilogue(pk, pidx, K++);
        if (!ok) break;
      }
      pk = ik;
      pidx = idx;
    }
    if (ok && pk >= 0) ok = epilogue(pk, pidx, K++);
  }
  tc_fence_before();
  __syncthreads();
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

}  // namespace

bool tc_supported(const mf_retrieve_desc& d) {
  if (d.flags & MF_RETRIEVE_FORCE_SIMT) return false;
  if (d.map_dtype != MF_BF16 || d.v_dtype != MF_BF16) return false;
  if (!(d.B == 64 || d.B == 128) || d.d != D) return false;
  if (d.h_kv <= 0 || d.h_r % d.h_kv != 0 || d.h_r / d.h_kv > GQP) return false;
  if (d.h_s <= 0 || d.h_s > 64) return false;
  if (d.paged && !(d.page_size == 8 || d.page_size == 16 || d.page_size == 32 || d.page_size == 64))
    return false;
  if (!d.paged && d.total_k >= (int64_t)1 << 31) return false;
  return true;
}

bool launch_retrieve_tc(const mf_retrieve_desc* const* ds, const RetrieveLayer* ls, int n,
                        uint32_t* status, cudaStream_t st, std::string* err, bool first) {
  if (n < 1 || n > NRMAX) { *err = "1 to 4 receivers per launch"; return false; }
  const mf_retrieve_desc& d0 = *ds[0];
  const RetrieveLayer& l0 = ls[0];
  const int B = d0.B;
  CUtensorMap tmA;
  {  // kept blocks [capacity][h_s][B][B]: dims (key j, sender head s, row i, block n)
    const uint64_t dims[4] = {(uint64_t)B, (uint64_t)d0.h_s, (uint64_t)B,
                              (uint64_t)std::max<int64_t>(l0.capacity, 1)};
    const uint64_t strides[3] = {(uint64_t)B * B * 2, (uint64_t)B * 2, (uint64_t)d0.h_s * B * B * 2};
    const uint32_t box[4] = {KT, SC, R, 1};
    if (!encode(&tmA, l0.values, 4, dims, strides, box, err)) return false;
  }
  VMaps vm;
  memset(&vm, 0, sizeof vm);
  TcParams p{};
  p.row_ptr = l0.row_ptr; p.col_idx = l0.col_idx; p.capacity = l0.capacity;
  p.cu_q = d0.cu_seqlens_q; p.cu_k = d0.cu_seqlens_k; p.qblock_base = d0.qblock_base;
  p.nqbq = (d0.max_seqlen_q + B - 1) / B;
  p.rcs = B / R;
  p.h_s = d0.h_s; p.nsc = (d0.h_s + SC - 1) / SC; p.B = B;
  p.nrecv = n;
  p.status = status;
  p.wait_ns = wait_limit_ns();
  p.stall = wait_stall();
  p.dep_wait = first ? 1 : 0;
  int NH = 0;
  for (int k = 0; k < n; ++k) {
    const mf_retrieve_desc& d = *ds[k];
    const RetrieveLayer& l = ls[k];
    // a box: 64 dims x the rows x 2 kv heads x 2 d halves, landing as [d half][head][row]
    if (!d.paged) {  // V [T][h_kv][d]: dims (dim in half, token, kv head, d half)
      const uint64_t dims[4] = {64, (uint64_t)std::max<int64_t>(d.total_k, 1), (uint64_t)d.h_kv, 2};
      const uint64_t strides[3] = {(uint64_t)d.h_kv * D * 2, (uint64_t)D * 2, 128};
      const uint32_t box[4] = {64, KT, 2, 2};
      if (!encode(&vm.m[k], l.V, 4, dims, strides, box, err)) return false;
    } else {  // V [pages][page][h_kv][d]: dims (dim in half, row in page, kv head, d half, page)
      const uint64_t dims[5] = {64, (uint64_t)d.page_size, (uint64_t)d.h_kv, 2,
                                (uint64_t)std::max(d.n_pages, 1)};
      const uint64_t strides[4] = {(uint64_t)d.h_kv * D * 2, (uint64_t)D * 2, 128,
                                   (uint64_t)d.page_size * d.h_kv * D * 2};
      const uint32_t box[5] = {64, (uint32_t)d.page_size, 2, 2, 1};
      if (!encode(&vm.m[k], l.V, 5, dims, strides, box, err)) return false;
    }
    RecvParams& r = p.rv[k];
    r.W = l.W; r.O = l.O;
    r.o_f32 = (d.flags & MF_RETRIEVE_O_F32) ? 1 : 0;
    r.p_split = (d.flags & MF_RETRIEVE_P_SPLIT) ? 1 : 0;
    r.block_table = d.block_table; r.paged = d.paged; r.page_size = d.page_size;
    r.n_pages = d.n_pages; r.max_pages = d.max_pages; r.total_k = (int)d.total_k;
    r.h_r = d.h_r; r.h_kv = d.h_kv; r.gq = d.h_r / d.h_kv;
    r.hcs = (d.h_kv + NG - 1) / NG;
    p.hh_base[k] = NH;
    NH += r.hcs;
  }
  p.hh_base[n] = NH;
  p.NH = NH;
  const int64_t n_items = (int64_t)d0.nseq * p.nqbq * p.rcs * NH;
  if (n_items == 0) return true;
  if (n_items >= ((int64_t)1 << 31)) { *err = "too many work items"; return false; }
  p.n_items = (int)n_items;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // persistent grid, a multiple of the head-chunk count (one receiver and one W^T per CTA)
  int64_t grid = std::min<int64_t>(n_items, sms);
  grid = std::max<int64_t>(NH, grid / NH * NH);
  cudaError_t e = cudaFuncSetAttribute(k_retrieve_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k_retrieve_tc, tmA, vm, p);
  if (e != cudaSuccess) { *err = cudaGetErrorString(e); return false; }
  e = cudaGetLastError();
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
