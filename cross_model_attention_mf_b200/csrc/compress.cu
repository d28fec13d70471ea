// Block-sparse compression of one sender layer's attention maps.
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com),
// section "存不下、读得慢?三个工程优化手段", subsection 1 "只存重要的:块稀疏压缩":
// the map is cut into regular 2-D blocks; block-level statistics are computed
// first, then the blocks to keep are chosen by cumulative attention probability,
// and only those are written -- no second dense matrix is assembled.
//
// Kernels (one launch each, all on the caller's stream):
//   k_meta          per-sequence geometry of the varlen pack (one thread); the grid
//                   clears the selection's look-back flags
//   k_stats         head-summed mass of every causal block: a streaming reduction
//                   with 16-byte loads, float32 partials of 8 (bf16) or 4 (f32)
//                   elements combined in float64, fixed order (deterministic)
//   k_select        per query block: sort candidates (mass desc, kb asc), walk
//                   the running float64 sum until it reaches tau * total; the row's
//                   offset by a decoupled look-back over the earlier rows' counts,
//                   then its kept indices in ascending order into col_idx
//   k_gather        copy each kept block with the causal/length mask applied, one
//                   (block, sender head) unit per CTA iteration
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "mf_internal.cuh"

namespace mfi {
namespace {

constexpr int META_HDR = 4;

__device__ inline int find_seq(const int64_t* meta, int nseq, int64_t x, int field) {
  // last s with meta[seq s].field <= x (fields are non-decreasing in s)
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (meta[META_HDR + 4 * mid + field] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ inline int tri_row(int64_t c) {
  int q = (int)((sqrt(8.0 * (double)c + 1.0) - 1.0) * 0.5);
  while ((int64_t)(q + 1) * (q + 2) / 2 <= c) ++q;
  while ((int64_t)q * (q + 1) / 2 > c) --q;
  return q;
}

// The varlen pack's geometry: header (total rows, total causal blocks, selection ticket = 0, -)
// and per sequence (L, nqb, row_base, cb_base), from its cu_seqlens (cu) and map offsets (off,
// may be null; a(s) = off[s] * elem_bytes must be 16-byte aligned).  One thread; returns the
// status bits of invalid sequences (which count as empty).
__device__ __noinline__ uint32_t meta_fill(const int32_t* cu, const int64_t* off, int nseq, int max_seqlen,
                              int B, int elem_bytes, int64_t* meta) {
  int64_t rows = 0, cb = 0;
  uint32_t st = 0;
  for (int s = 0; s < nseq; ++s) {
    int64_t L = (int64_t)cu[s + 1] - cu[s];
    if (L < 0 || L > max_seqlen) { st |= ST_INDEX; L = 0; }
    if (off && ((off[s] * elem_bytes) % 16 != 0 || off[s] < 0)) { st |= ST_ALIGN; L = 0; }
    const int64_t nqb = (L + B - 1) / B;
    int64_t* m = meta + META_HDR + 4 * s;
    m[0] = L; m[1] = nqb; m[2] = rows; m[3] = cb;
    rows += nqb;
    cb += nqb * (nqb + 1) / 2;
  }
  meta[0] = rows; meta[1] = cb; meta[2] = 0; meta[3] = 0;  // meta[2]: selection ticket
  return st;
}

__global__ void k_meta(const int32_t* cu, const int64_t* off, int nseq, int max_seqlen, int B,
                       int elem_bytes, int64_t* meta, uint32_t* status, int32_t* row_ptr,
                       int32_t* nnz_out, unsigned long long* flags, int64_t max_rows) {
  // the selection's look-back flags start cleared (every thread of the grid)
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < max_rows;
       r += (int64_t)gridDim.x * blockDim.x)
    flags[r] = 0ull;
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  const uint32_t st = meta_fill(cu, off, nseq, max_seqlen, B, elem_bytes, meta);
  if (meta[0] == 0) {  // no query block at all: an empty BSR
    row_ptr[0] = 0;
    *nnz_out = 0;
  }
  if (st) atomicOr(status, st);
}

template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int EPV = 4;
  __device__ static float get(const uint4& v, int e) {
    const uint32_t w = e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
    return __uint_as_float(w);
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int EPV = 8;
  __device__ static float get(const uint4& v, int e) {
    const uint32_t w = (e >> 1) == 0 ? v.x : (e >> 1) == 1 ? v.y : (e >> 1) == 2 ? v.z : v.w;
    return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};

template <int NT>
__device__ inline double block_sum_f64(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int k = 0; k < NT / 32; ++k) t += red[k];
  __syncthreads();
  return t;  // valid in thread 0
}

// Geometry computed inside k_stats (no k_meta launch) for batches of up to this many sequences
// and blocks of up to 64: measured faster there (Ministral-like pair: -3 us per call); with
// B = 128 the inlined pass changed k_stats' register allocation and cost ~17 us on the
// long-context case, so that size keeps the separate launch
constexpr int INLINE_META_SEQ = 64;
inline bool inline_meta_for(int nseq, int B) { return nseq <= INLINE_META_SEQ && B <= 64; }
struct MetaIn {           // k_stats computes the geometry itself when inline_meta is set
  const int32_t* cu;
  int max_seqlen, elem_bytes, inline_meta;
  int64_t* meta_out;      // written by CTA 0
  uint32_t* status;
  int32_t* row_ptr;       // empty batch: row_ptr[0] = 0
  int32_t* nnz_out;
  unsigned long long* flags;  // cleared by the grid
  int64_t max_rows;
};

// Masses of every causal block.  Item = (sequence, qb, kb) over all sender heads.
template <typename T, int B, int NT>
__global__ void __launch_bounds__(NT) k_stats(const T* __restrict__ maps,
                                              const int64_t* __restrict__ seq_off,
                                              const int64_t* __restrict__ meta_g, int nseq,
                                              int h_s, double* __restrict__ mass, MetaIn mi) {
  constexpr int EPV = Vec<T>::EPV, VPR = B / EPV, VPB = B * VPR;  // vectors per row / per head
  constexpr int U = 4;
  __shared__ double red[NT / 32];
  __shared__ int64_t s_meta[META_HDR + 4 * INLINE_META_SEQ];
  __shared__ int32_t s_cu[INLINE_META_SEQ + 1];
  __shared__ int64_t s_off[INLINE_META_SEQ];
  const int64_t* meta = meta_g;
  // (compiled for B <= 64 only: see inline_meta_for)
  if constexpr (B <= 64) {
    if (mi.inline_meta) {
      // the selection's look-back flags start cleared (every thread of the grid)
      for (int64_t r = (int64_t)blockIdx.x * NT + threadIdx.x; r < mi.max_rows;
           r += (int64_t)gridDim.x * NT)
        mi.flags[r] = 0ull;
      // every CTA computes the geometry into shared memory (warp 0 loads the inputs, thread 0
      // runs the sums); CTA 0 also publishes it for the later passes
      if (threadIdx.x < 32) {
        for (int k = threadIdx.x; k <= nseq; k += 32) s_cu[k] = mi.cu[k];
        if (seq_off)
          for (int k = threadIdx.x; k < nseq; k += 32) s_off[k] = seq_off[k];
        __syncwarp();
        if (threadIdx.x == 0) {
          const uint32_t st = meta_fill(s_cu, seq_off ? s_off : nullptr, nseq, mi.max_seqlen, B,
                                        mi.elem_bytes, s_meta);
          if (blockIdx.x == 0) {
            for (int k = 0; k < META_HDR + 4 * nseq; ++k) mi.meta_out[k] = s_meta[k];
            if (s_meta[0] == 0) {  // no query block at all: an empty BSR
              mi.row_ptr[0] = 0;
              *mi.nnz_out = 0;
            }
            if (st) atomicOr(mi.status, st);
          }
        }
      }
      __syncthreads();
      meta = s_meta;
    }
  }
  const int64_t total = meta[1];
  const int64_t nv = (int64_t)h_s * VPB;
  for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
    const int s = find_seq(meta, nseq, item, 3);
    const int64_t* m = meta + META_HDR + 4 * s;
    const int64_t L = m[0], Lp = m[1] * B, c = item - m[3];
    const int qb = tri_row(c);
    const int kb = (int)(c - (int64_t)qb * (qb + 1) / 2);
    const T* base = maps + seq_off[s];
    const bool full = kb < qb && (int64_t)(qb + 1) * B <= L;
    double acc = 0.0;
    for (int64_t v0 = threadIdx.x; v0 < nv; v0 += (int64_t)NT * U) {
      uint4 r[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t v = v0 + (int64_t)u * NT;
        if (v < nv) {
          const int64_t hs = v / VPB;
          const int rem = (int)(v - hs * VPB);
          const int ii = rem / VPR, jv = rem % VPR;
          const T* p = base + ((hs * Lp) + (int64_t)qb * B + ii) * Lp + (int64_t)kb * B + jv * EPV;
          r[u] = __ldg(reinterpret_cast<const uint4*>(p));
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t v = v0 + (int64_t)u * NT;
        if (v < nv) {
          float part = 0.0f;
          if (full) {
            float a[EPV];
#pragma unroll
            for (int e = 0; e < EPV; ++e) a[e] = Vec<T>::get(r[u], e);
            if constexpr (EPV == 8)
              part = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
            else
              part = (a[0] + a[1]) + (a[2] + a[3]);
          } else {
            const int64_t hs = v / VPB;
            const int rem = (int)(v - hs * VPB);
            const int ii = rem / VPR, jv = rem % VPR;
            const int64_t i = (int64_t)qb * B + ii;
#pragma unroll
            for (int e = 0; e < EPV; ++e) {
              const int64_t j = (int64_t)kb * B + jv * EPV + e;
              if (i < L && j <= i) part += Vec<T>::get(r[u], e);
            }
          }
          acc += (double)part;
        }
      }
    }
    const double t = block_sum_f64<NT>(acc, red);
    if (threadIdx.x == 0) mass[item] = t;
  }
}

__device__ inline uint64_t order_key(double x) {
  if (x == 0.0) x = 0.0;  // -0 sorts with +0
  const uint64_t b = (uint64_t)__double_as_longlong(x);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
// the mass a key was made from (bit for bit; -0 comes back as +0)
__device__ inline double key_mass(uint64_t k) {
  return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

// One CTA per query block (row).  Candidates kb < qb sorted by (mass desc, kb asc); the walk
// starts from the diagonal block.  The row's place in col_idx comes from a decoupled look-back
// (single-pass prefix sum): rows are numbered by a ticket taken when the CTA starts (meta[2]),
// so every earlier row is already running; each row publishes its count (FLAG_AGG), sums the
// counts or the inclusive prefix (FLAG_PREFIX) of the rows before it, publishes its own
// inclusive prefix and writes its kept blocks into col_idx / kept_row and its row_ptr entry.
// The flags were cleared by k_meta.  Waiting for an earlier row's flag is bounded by wait_ns.
constexpr unsigned long long FLAG_AGG = 1ull << 62, FLAG_PREFIX = 1ull << 63,
                             FLAG_VALUE = (1ull << 62) - 1;
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
template <int NT>
__global__ void __launch_bounds__(NT) k_select(int64_t* __restrict__ meta, int nseq,
                                               const double* __restrict__ mass, double tau,
                                               unsigned long long* __restrict__ flags,
                                               int32_t* __restrict__ row_ptr,
                                               int32_t* __restrict__ col_idx,
                                               int32_t* __restrict__ kept_row,
                                               int32_t* __restrict__ nnz_out, int64_t capacity,
                                               uint32_t* status, uint64_t wait_ns) {
  extern __shared__ uint64_t sm[];
  __shared__ int s_nkeep;
  __shared__ int64_t s_row, s_base;
  // launched as a programmatic dependent of the block-mass pass: wait until that grid has
  // completed and its writes are visible (returns at once after an ordinary launch); the gather
  // may then be launched, and waits for this grid in turn
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0)
    s_row = (int64_t)atomicAdd(reinterpret_cast<unsigned long long*>(meta + 2), 1ull);
  __syncthreads();
  const int64_t row = s_row;
  const int64_t R = meta[0];
  if (row >= R) return;
  const int s = find_seq(meta, nseq, row, 2);
  const int64_t* m = meta + META_HDR + 4 * s;
  const int qb = (int)(row - m[2]);
  const int64_t tri = m[3] + (int64_t)qb * (qb + 1) / 2;
  const double* mr = mass + tri;
  const int n = qb;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  uint64_t* key = sm;
  int* idx = reinterpret_cast<int*>(sm + n2);
  for (int t = threadIdx.x; t < n2; t += NT) {
    if (t < n) { key[t] = order_key(mr[t]); idx[t] = t; }
    else { key[t] = 0ull; idx[t] = 0x7fffffff; }
  }
  __syncthreads();
  // bitonic sort into (key desc, idx asc)
  for (int k = 2; k <= n2; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n2; t += NT) {
        const int p = t ^ j;
        if (p > t) {
          const bool up = (t & k) == 0;  // this run sorts into the target order
          const uint64_t ka = key[t], kb2 = key[p];
          const int ia = idx[t], ib = idx[p];
          const bool a_first = ka > kb2 || (ka == kb2 && ia < ib);
          if (up != a_first) {
            key[t] = kb2; key[p] = ka; idx[t] = ib; idx[p] = ia;
          }
        }
      }
      __syncthreads();
    }
  if (threadIdx.x == 0) {
    // the walk reads the candidates' masses back from their sorted keys (independent shared
    // loads; only the float64 sums form a chain)
    const double diag = mr[qb];
    double total = 0.0;
    total += diag;
    for (int t = 0; t < n; ++t) total += key_mass(key[t]);
    const double target = tau * total;
    double S = 0.0;
    int nk = n + 1;
    S += diag;
    if (S >= target) {
      nk = 1;
    } else {
      for (int t = 0; t < n; ++t) {
        S += key_mass(key[t]);
        if (S >= target) { nk = t + 2; break; }
      }
    }
    s_nkeep = nk;
  }
  __syncthreads();
  const int nk = s_nkeep;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // publish this row's count, then find its offset from the rows before it
  if (threadIdx.x == 0) {
    const unsigned long long w = FLAG_AGG | (unsigned long long)nk;
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(flags + row), "l"(w) : "memory");
  }
  if (warp == 0) {
    int64_t prefix = 0;
    int64_t j0 = row - 1;  // lane l reads row j0 - l; rows before 0 count as a prefix of 0
    const uint64_t t0 = gtime();
    while (true) {
      const int64_t j = j0 - lane;
      unsigned long long f = FLAG_PREFIX;
      if (j >= 0) asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(f) : "l"(flags + j) : "memory");
      if (!__all_sync(0xffffffffu, f != 0ull)) {  // an earlier row has not published yet
        if (gtime() - t0 > wait_ns) {
          if (lane == 0) atomicOr(status, ST_TIMEOUT);
          break;
        }
        continue;
      }
      const uint32_t pre = __ballot_sync(0xffffffffu, (f & FLAG_PREFIX) != 0ull);
      const int first = pre ? __ffs(pre) - 1 : 31;  // nearest row holding an inclusive prefix
      int64_t v = lane <= first ? (int64_t)(f & FLAG_VALUE) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      prefix += v;
      if (pre) break;
      j0 -= 32;
    }
    if (lane == 0) {
      s_base = prefix;
      const unsigned long long w = FLAG_PREFIX | (unsigned long long)(prefix + nk);
      asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(flags + row), "l"(w) : "memory");
      row_ptr[row] = (int32_t)prefix;
      if (row == R - 1) {
        row_ptr[R] = (int32_t)(prefix + nk);
        *nnz_out = (int32_t)(prefix + nk);
        if (prefix + nk > capacity) atomicOr(status, ST_CAPACITY);
      }
    }
  }
  // kept flags by key-block index (reusing the key array), then an ordered compaction into
  // col_idx[base ...] (ascending key blocks), skipping entries past the capacity
  uint8_t* kept = reinterpret_cast<uint8_t*>(key);
  for (int t = threadIdx.x; t <= n; t += NT) kept[t] = 0;
  __syncthreads();
  for (int t = threadIdx.x; t < nk - 1; t += NT) kept[idx[t]] = 1;
  if (threadIdx.x == 0) kept[qb] = 1;
  __syncthreads();
  const int64_t base = s_base;
  __shared__ int s_warp[NT / 32];
  __shared__ int s_cnt;
  if (threadIdx.x == 0) s_cnt = 0;
  for (int k0 = 0; k0 <= n; k0 += NT) {
    const int kb = k0 + threadIdx.x;
    const bool f = kb <= n && kept[kb];
    const uint32_t bal = __ballot_sync(0xffffffffu, f);
    __syncthreads();
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    int before = s_cnt;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    const int64_t e = base + before + __popc(bal & ((1u << lane) - 1u));
    if (f && e < capacity) {
      col_idx[e] = kb;
      kept_row[e] = (int32_t)row;
    }
    __syncthreads();
    if (threadIdx.x == 0)
      for (int w = 0; w < NT / 32; ++w) s_cnt += s_warp[w];
  }
}

template <typename T, int B, int NT>
__global__ void __launch_bounds__(NT) k_gather(const T* __restrict__ maps,
                                               const int64_t* __restrict__ seq_off,
                                               const int64_t* __restrict__ meta, int nseq,
                                               int h_s, const int32_t* __restrict__ nnz_in,
                                               int64_t capacity,
                                               const int32_t* __restrict__ col_idx,
                                               const int32_t* __restrict__ kept_row,
                                               T* __restrict__ values) {
  constexpr int EPV = Vec<T>::EPV, VPR = B / EPV, VPB = B * VPR;  // vectors per row / per head
  constexpr int U = (VPB + NT - 1) / NT;
  // launched as a programmatic dependent of the selection: wait for its writes
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t nnz = min((int64_t)*nnz_in, capacity);
  const int64_t units = nnz * h_s;
  for (int64_t u0 = blockIdx.x; u0 < units; u0 += gridDim.x) {
    const int64_t n = u0 / h_s;
    const int hs = (int)(u0 - n * h_s);
    const int64_t row = kept_row[n];
    const int kb = col_idx[n];
    const int s = find_seq(meta, nseq, row, 2);
    const int64_t* m = meta + META_HDR + 4 * s;
    const int64_t L = m[0], Lp = m[1] * B;
    const int qb = (int)(row - m[2]);
    const T* src = maps + seq_off[s] + ((int64_t)hs * Lp + (int64_t)qb * B) * Lp + (int64_t)kb * B;
    uint4* dst = reinterpret_cast<uint4*>(values + (n * h_s + hs) * (int64_t)B * B);
    const bool full = kb < qb && (int64_t)(qb + 1) * B <= L;
    uint4 r[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int v = threadIdx.x + k * NT;
      if (v < VPB) {
        const int ii = v / VPR, jv = v % VPR;
        r[k] = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)ii * Lp + jv * EPV));
        if (!full) {
          const int64_t i = (int64_t)qb * B + ii;
          uint32_t w[4] = {r[k].x, r[k].y, r[k].z, r[k].w};
#pragma unroll
          for (int e = 0; e < EPV; ++e) {
            const int64_t j = (int64_t)kb * B + jv * EPV + e;
            if (!(i < L && j <= i)) {
              if (EPV == 4) w[e] = 0u;
              else w[e >> 1] &= (e & 1) ? 0x0000ffffu : 0xffff0000u;
            }
          }
          r[k] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int v = threadIdx.x + k * NT;
      if (v < VPB) __stcs(dst + v, r[k]);
    }
  }
}

// a launch that may start while the previous kernel on the stream drains (programmatic
// dependent launch); the kernel waits (griddepcontrol.wait) before reading that kernel's output
void dependent_launch(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* at, int grid, int block,
                      size_t smem, cudaStream_t st) {
  cfg->gridDim = dim3((unsigned)grid);
  cfg->blockDim = dim3((unsigned)block);
  cfg->dynamicSmemBytes = smem;
  cfg->stream = st;
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg->attrs = at;
  cfg->numAttrs = 1;
}

template <typename T, int B>
cudaError_t launch_typed(const mf_compress_desc& d, const CompressWs& ws, uint32_t* status,
                         cudaStream_t st, int sms) {
  constexpr int NT = 256;
  const T* maps = static_cast<const T*>(d.maps);
  double* mass = d.block_mass_out ? d.block_mass_out : ws.mass;
  const int grid_stats = (int)std::min<int64_t>(ws.max_cb, (int64_t)sms * 8);
  MetaIn mi{};
  if (inline_meta_for(d.nseq, B)) {
    mi.cu = d.cu_seqlens; mi.max_seqlen = d.max_seqlen; mi.elem_bytes = (int)sizeof(T);
    mi.inline_meta = 1; mi.meta_out = ws.meta; mi.status = status; mi.row_ptr = d.row_ptr;
    mi.nnz_out = d.nnz_out; mi.flags = ws.flags; mi.max_rows = ws.max_rows;
  }
  k_stats<T, B, NT><<<grid_stats, NT, 0, st>>>(maps, d.map_seq_offset, ws.meta, d.nseq, d.h_s,
                                                mass, mi);
  cudaError_t e = launch_select(ws, d.nseq, d.max_seqlen, B, mass, d.tau, d.row_ptr, d.col_idx,
                                d.nnz_out, d.capacity_blocks, status, st);
  if (e != cudaSuccess) return e;
  const int grid_g = (int)std::max<int64_t>(
      1, std::min<int64_t>(std::max<int64_t>(d.capacity_blocks, 1) * d.h_s, (int64_t)sms * 8));
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute at[1];
  dependent_launch(&cfg, at, grid_g, NT, 0, st);
  return cudaLaunchKernelEx(&cfg, k_gather<T, B, NT>, maps, d.map_seq_offset,
                            (const int64_t*)ws.meta, d.nseq, d.h_s, (const int32_t*)d.nnz_out,
                            d.capacity_blocks, (const int32_t*)d.col_idx,
                            (const int32_t*)ws.kept_row, static_cast<T*>(d.values));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

cudaError_t launch_meta(const int32_t* cu, const int64_t* off, int nseq, int max_seqlen, int B,
                        int elem_bytes, const CompressWs& ws, uint32_t* status, int32_t* row_ptr,
                        int32_t* nnz_out, cudaStream_t st) {
  const int grid = (int)std::min<int64_t>(std::max<int64_t>((ws.max_rows + 255) / 256, 1), 1024);
  k_meta<<<grid, 256, 0, st>>>(cu, off, nseq, max_seqlen, B, elem_bytes, ws.meta, status, row_ptr,
                               nnz_out, ws.flags, ws.max_rows);
  return cudaGetLastError();
}

cudaError_t launch_select(const CompressWs& ws, int nseq, int max_seqlen, int B, const double* mass,
                          double tau, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                          int64_t capacity, uint32_t* status, cudaStream_t st) {
  const int64_t nqb_max = (max_seqlen + B - 1) / B;
  int n2 = 1;
  while (n2 < nqb_max) n2 <<= 1;
  const size_t smem_sel = (size_t)n2 * (sizeof(uint64_t) + sizeof(int));
  if (smem_sel > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_select<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_sel);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute at[1];
  dependent_launch(&cfg, at, (int)std::max<int64_t>(ws.max_rows, 1), 128, smem_sel, st);
  return cudaLaunchKernelEx(&cfg, k_select<128>, ws.meta, nseq, mass, tau, ws.flags, row_ptr,
                            col_idx, ws.kept_row, nnz_out, capacity, status, wait_limit_ns());
}

size_t compress_ws_layout(const mf_compress_desc& d, CompressWs* ws, void* base) {
  const int64_t nqb_max = (d.max_seqlen + d.B - 1) / d.B;
  const int64_t max_rows = (int64_t)d.nseq * nqb_max;
  const int64_t max_cb = (int64_t)d.nseq * nqb_max * (nqb_max + 1) / 2;
  size_t off = 0;
  const size_t o_meta = off; off = align_up(off + sizeof(int64_t) * (META_HDR + 4 * (size_t)d.nseq), 256);
  const size_t o_mass = off; off = align_up(off + sizeof(double) * (size_t)max_cb, 256);
  const size_t o_flags = off; off = align_up(off + sizeof(uint64_t) * (size_t)std::max<int64_t>(max_rows, 1), 256);
  const size_t o_kept = off; off = align_up(off + sizeof(int32_t) * (size_t)std::max<int64_t>(d.capacity_blocks, 1), 256);
  if (ws) {
    char* b = static_cast<char*>(base);
    ws->meta = reinterpret_cast<int64_t*>(b + o_meta);
    ws->mass = reinterpret_cast<double*>(b + o_mass);
    ws->flags = reinterpret_cast<unsigned long long*>(b + o_flags);
    ws->kept_row = reinterpret_cast<int32_t*>(b + o_kept);
    ws->max_cb = max_cb;
    ws->max_rows = max_rows;
  }
  return off;
}

cudaError_t launch_compress(const mf_compress_desc& d, const CompressWs& ws, uint32_t* status,
                            cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int elem = d.dtype == MF_F32 ? 4 : 2;
  // the geometry pass: inside k_stats where inline_meta_for says so, else its own launch (also
  // when there is no query block at all and k_stats does not run)
  if (!inline_meta_for(d.nseq, d.B) || ws.max_cb == 0) {
    cudaError_t e = launch_meta(d.cu_seqlens, d.map_seq_offset, d.nseq, d.max_seqlen, d.B, elem,
                                ws, status, d.row_ptr, d.nnz_out, st);
    if (e != cudaSuccess) return e;
  }
  if (ws.max_cb == 0) return cudaSuccess;  // no query block (max_seqlen 0): k_meta wrote the empty BSR
  if (d.dtype == MF_F32) {
    if (d.B == 32) return launch_typed<float, 32>(d, ws, status, st, sms);
    if (d.B == 64) return launch_typed<float, 64>(d, ws, status, st, sms);
    return launch_typed<float, 128>(d, ws, status, st, sms);
  }
  if (d.B == 32) return launch_typed<__nv_bfloat16, 32>(d, ws, status, st, sms);
  if (d.B == 64) return launch_typed<__nv_bfloat16, 64>(d, ws, status, st, sms);
  return launch_typed<__nv_bfloat16, 128>(d, ws, status, st, sms);
}

}  // namespace mfi
