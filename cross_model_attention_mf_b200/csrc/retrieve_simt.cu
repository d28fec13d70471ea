// Fused map retrieval, float32 SIMT kernel.
//
// Serves float32 maps (tensor-core float32 would be TF32 and miss a 1e-5
// tolerance) and every shape the tcgen05 kernel does not cover.  Same
// computation as the tensor-core path (MapFlow page "MapFlow开源:大模型换班,
// Prefill为何能快20%?", section "存不下、读得慢?三个工程优化手段", subsection 3
// "算得省的:融合内核执行"): per kept block, the receiver head's map tile
// P = sum_s W[r][s] A_s is formed in shared memory and P.V is accumulated in
// registers; the dense receiver map is never written.
//
// CTA = (sequence, query block of the chunk, receiver head), 256 threads.
#include <cuda_bf16.h>
#include <stdint.h>

#include "mf_internal.cuh"

namespace mfi {
namespace {

constexpr int NT = 256;
constexpr int MAX_ACC = 64;  // B * d / NT <= 64

template <typename T> __device__ inline float ld(const T* p);
template <> __device__ inline float ld<float>(const float* p) { return __ldg(p); }
template <> __device__ inline float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ inline void st(T* p, float v);
template <> __device__ inline void st<float>(float* p, float v) { *p = v; }
template <> __device__ inline void st<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

struct SimtParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const void* values;
  int64_t capacity;
  const float* W;  // [h_r][h_s]
  const void* V;
  void* O;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* qblock_base;
  const int32_t* block_table;
  int paged, page_size, n_pages, max_pages;
  int64_t total_k;
  int nqbq, h_s, B, h_r, h_kv, d;
  uint32_t* status;
};

template <typename TA, typename TV>
__global__ void __launch_bounds__(NT) k_retrieve_simt(SimtParams p) {
  extern __shared__ float sm[];
  float* P = sm;                        // [B][B]
  float* Vt = P + p.B * p.B;            // [B][d]
  float* Ws = Vt + p.B * p.d;           // [h_s]
  const int B = p.B, d = p.d;
  int64_t item = blockIdx.x;
  const int r = (int)(item % p.h_r);
  item /= p.h_r;
  const int qbl = (int)(item % p.nqbq);
  const int s = (int)(item / p.nqbq);
  const int q_len = p.cu_q[s + 1] - p.cu_q[s];
  const int k_len = p.cu_k[s + 1] - p.cu_k[s];
  const int q0 = k_len - q_len;
  if (q_len <= 0 || q0 < 0) return;
  const int qb = q0 / B + qbl;
  if ((int64_t)qb * B >= k_len) return;
  const int row_lo = max(q0, qb * B), row_hi = min(k_len, qb * B + B);
  const int64_t brow = (int64_t)p.qblock_base[s] + qb;
  int64_t rp0 = p.row_ptr[brow], rp1 = p.row_ptr[brow + 1];
  if (rp0 < 0 || rp1 < rp0 || rp1 > p.capacity || rp1 - rp0 > qb + 1) {
    if (threadIdx.x == 0) atomicOr(p.status, ST_INDEX);
    rp1 = rp0;  // outputs become zeros
  }
  const int g = (int)(((int64_t)r * p.h_kv) / p.h_r);
  for (int t = threadIdx.x; t < p.h_s; t += NT) Ws[t] = p.W[(int64_t)r * p.h_s + t];
  const int nown = (B * d + NT - 1) / NT;
  float acc[MAX_ACC];
#pragma unroll
  for (int k = 0; k < MAX_ACC; ++k) acc[k] = 0.0f;
  __syncthreads();
  const TA* vals = static_cast<const TA*>(p.values);
  const TV* V = static_cast<const TV*>(p.V);
  for (int64_t e = rp0; e < rp1; ++e) {
    const int kb = p.col_idx[e];
    if (kb < 0 || kb > qb) {
      if (threadIdx.x == 0) atomicOr(p.status, ST_INDEX);
      continue;
    }
    const TA* blk = vals + e * (int64_t)p.h_s * B * B;
    for (int t = threadIdx.x; t < B * B; t += NT) {
      const int ii = t / B, jj = t % B;
      float pv = 0.0f;
      if (kb * B + jj <= qb * B + ii)
        for (int hs = 0; hs < p.h_s; ++hs) pv = fmaf(Ws[hs], ld<TA>(blk + (int64_t)hs * B * B + t), pv);
      P[t] = pv;
    }
    for (int t = threadIdx.x; t < B * d; t += NT) {
      const int jj = t / d, c = t % d;
      const int tok = kb * B + jj;
      float v = 0.0f;
      if (tok < k_len) {
        if (p.paged) {
          const int slot = tok / p.page_size;
          const int page = slot < p.max_pages ? p.block_table[(int64_t)s * p.max_pages + slot] : -1;
          if (page >= 0 && page < p.n_pages)
            v = ld<TV>(V + (((int64_t)page * p.page_size + tok % p.page_size) * p.h_kv + g) * d + c);
          else
            atomicOr(p.status, ST_PAGE);
        } else {
          const int64_t row = (int64_t)p.cu_k[s] + tok;
          if (row < p.total_k) v = ld<TV>(V + (row * p.h_kv + g) * d + c);
        }
      }
      Vt[t] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < MAX_ACC; ++k) {
      if (k < nown) {
        const int o = threadIdx.x + k * NT;
        if (o < B * d) {
          const int ii = o / d, c = o % d;
          float a = acc[k];
          for (int jj = 0; jj < B; ++jj) a = fmaf(P[ii * B + jj], Vt[jj * d + c], a);
          acc[k] = a;
        }
      }
    }
    __syncthreads();
  }
  TV* O = static_cast<TV*>(p.O);
#pragma unroll
  for (int k = 0; k < MAX_ACC; ++k) {
    if (k < nown) {
      const int o = threadIdx.x + k * NT;
      if (o < B * d) {
        const int ii = o / d, c = o % d;
        const int i = qb * B + ii;
        if (i >= row_lo && i < row_hi) {
          const int64_t orow = (int64_t)p.cu_q[s] + (i - q0);
          st<TV>(O + (orow * p.h_r + r) * d + c, acc[k]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_retrieve_simt(const mf_retrieve_desc& d, const RetrieveLayer& l,
                                 uint32_t* status, cudaStream_t st) {
  SimtParams p{};
  p.row_ptr = l.row_ptr; p.col_idx = l.col_idx; p.values = l.values; p.capacity = l.capacity;
  p.W = l.W; p.V = l.V; p.O = l.O;
  p.cu_q = d.cu_seqlens_q; p.cu_k = d.cu_seqlens_k; p.qblock_base = d.qblock_base;
  p.block_table = d.block_table; p.paged = d.paged; p.page_size = d.page_size;
  p.n_pages = d.n_pages; p.max_pages = d.max_pages; p.total_k = d.total_k;
  p.nqbq = (d.max_seqlen_q + d.B - 1) / d.B;
  p.h_s = d.h_s; p.B = d.B; p.h_r = d.h_r; p.h_kv = d.h_kv; p.d = d.d;
  p.status = status;
  const int64_t grid = (int64_t)d.nseq * p.nqbq * d.h_r;
  if (grid == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)d.B * d.B + (size_t)d.B * d.d + d.h_s);
  cudaError_t e;
  auto launch = [&](auto kern) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return;
    kern<<<(unsigned)grid, NT, smem, st>>>(p);
    e = cudaGetLastError();
  };
  const bool fa = d.map_dtype == MF_F32, fv = d.v_dtype == MF_F32;
  if (fa && fv) launch(k_retrieve_simt<float, float>);
  else if (fa) launch(k_retrieve_simt<float, __nv_bfloat16>);
  else if (fv) launch(k_retrieve_simt<__nv_bfloat16, float>);
  else launch(k_retrieve_simt<__nv_bfloat16, __nv_bfloat16>);
  return e;
}

}  // namespace mfi
