// Seeded synthetic inputs on the GPU: sender attention maps and N(0,1) fills.
//
// Input generation only: nothing here computes block statistics, block
// selection, head mixing or P.V.  The recipe is the one written out in
// synth/maps.py (sink bonus, local decay, heavy columns, N(0,1) noise, causal
// row softmax), with its own implementation of the two published generators
// it needs:
//   SplitMix64 -- Steele, Lea, Flood, OOPSLA 2014 (counter form: the n-th
//                 output of the stream at `key` is mix64(key + (n+1)*GAMMA));
//   Box-Muller -- Box and Muller, Ann. Math. Stat. 1958, in float32 from two
//                 24-bit uniforms.
// CUDA's logf/cosf/sqrtf/expf are called, not re-derived.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace {

constexpr uint64_t GAMMA = 0x9E3779B97F4A7C15ull;
constexpr uint64_t TAG_NOISE = 1;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t tag, uint64_t a,
                                               uint64_t b, uint64_t c) {
  uint64_t k = seed;
  const uint64_t f[4] = {tag, a, b, c};
  for (int t = 0; t < 4; ++t) k = mix64(k ^ ((f[t] + 1) * GAMMA));
  return k;
}

__device__ inline uint64_t draw(uint64_t key, uint64_t n) { return mix64(key + (n + 1) * GAMMA); }

__device__ inline float normal01(uint64_t key, uint64_t n) {
  const uint64_t x0 = draw(key, 2 * n), x1 = draw(key, 2 * n + 1);
  const float u1 = ((float)(x0 >> 40) + 1.0f) * 0x1p-24f;
  const float u2 = (float)(x1 >> 40) * 0x1p-24f;
  const float r = sqrtf(-2.0f * logf(u1));
  return r * cosf(6.2831855f * u2);  // float32(2*pi)
}

struct RowCtx {
  uint64_t key;
  int i, Lp, reading;
  const uint32_t* heavy_bits;
};

__device__ inline float logit(const RowCtx& c, int j) {
  const bool sink = j < 4;
  const bool hv = (c.heavy_bits[j >> 5] >> (j & 31)) & 1u;
  const float bonus = 2.0f * (sink ? 1.0f : 0.0f) + 1.5f * (hv ? 1.0f : 0.0f);
  float decay = -0.05f * (float)(c.i - j);
  if (c.reading == 3 && (sink || hv)) decay = 0.0f;
  const float z = normal01(c.key, (uint64_t)c.i * (uint64_t)c.Lp + (uint64_t)j);
  return (bonus + decay) + z;
}

template <int NT>
__device__ inline float block_reduce(float v, bool is_max, float* red) {
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < NT / 32 ? red[lane] : (is_max ? -INFINITY : 0.0f);
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, w) : v + w;
    }
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

template <typename T>
__device__ inline void store(T* p, float v);
template <>
__device__ inline void store<float>(float* p, float v) { *p = v; }
template <>
__device__ inline void store<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// grid (Lp rows, h_s heads), NT threads: one causal softmax row per CTA.  Writes
// the row's entries up to the end of its diagonal block (the causal blocks);
// blocks above the diagonal are left untouched.
template <typename T, int NT>
__global__ void __launch_bounds__(NT) gen_maps_kernel(T* out, int L, int Lp, int B,
                                                       const int32_t* heavy, int n_heavy,
                                                       uint64_t seed, int layer, int seq,
                                                       int reading) {
  extern __shared__ uint32_t hbits[];
  __shared__ float red[32];
  const int i = blockIdx.x, s = blockIdx.y;
  const int nwords = (Lp + 31) / 32;
  for (int w = threadIdx.x; w < nwords; w += NT) hbits[w] = 0u;
  __syncthreads();
  for (int t = threadIdx.x; t < n_heavy; t += NT) {
    const int c = heavy[(size_t)s * n_heavy + t];
    if (c >= 0 && c < Lp) atomicOr(&hbits[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
  T* row = out + ((size_t)s * Lp + i) * (size_t)Lp;
  const int row_end = (i / B + 1) * B;
  if (i >= L) {
    for (int j = threadIdx.x; j < row_end; j += NT) store<T>(row + j, 0.0f);
    return;
  }
  RowCtx c{stream_key(seed, TAG_NOISE, (uint64_t)layer, (uint64_t)seq, (uint64_t)s), i, Lp,
           reading, hbits};
  float m = -INFINITY;
  for (int j = threadIdx.x; j <= i; j += NT) m = fmaxf(m, logit(c, j));
  m = block_reduce<NT>(m, true, red);
  float sum = 0.0f;
  for (int j = threadIdx.x; j <= i; j += NT) sum += expf(logit(c, j) - m);
  sum = block_reduce<NT>(sum, false, red);
  for (int j = threadIdx.x; j < row_end; j += NT)
    store<T>(row + j, j <= i ? expf(logit(c, j) - m) / sum : 0.0f);
}

template <typename T>
__global__ void fill_normal_kernel(T* out, int64_t n, uint64_t key, float scale) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    float z = normal01(key, (uint64_t)e);
    store<T>(out + e, scale == 1.0f ? z : z * scale);
  }
}

}  // namespace

extern "C" {

// dtype: 0 = float32, 1 = bfloat16.  Returns a cudaError_t value (0 = success).
int mfsynth_gen_maps(void* out, int dtype, int L, int Lp, int B, int h_s, const int32_t* heavy,
                     int n_heavy, unsigned long long seed, int layer, int seq, int reading,
                     void* stream) {
  if (!out || L < 0 || Lp < L || B <= 0 || Lp % B || h_s <= 0 || h_s > 65535) return 1;
  if (Lp == 0) return 0;
  constexpr int NT = 256;
  dim3 grid(Lp, h_s);
  const size_t smem = (size_t)((Lp + 31) / 32) * 4;
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype == 0)
    gen_maps_kernel<float, NT><<<grid, NT, smem, st>>>((float*)out, L, Lp, B, heavy, n_heavy,
                                                       seed, layer, seq, reading);
  else
    gen_maps_kernel<__nv_bfloat16, NT><<<grid, NT, smem, st>>>(
        (__nv_bfloat16*)out, L, Lp, B, heavy, n_heavy, seed, layer, seq, reading);
  return (int)cudaGetLastError();
}

int mfsynth_fill_normal(void* out, int dtype, long long n, unsigned long long key, float scale,
                        void* stream) {
  if (!out || n < 0) return 1;
  if (n == 0) return 0;
  cudaStream_t st = (cudaStream_t)stream;
  const int grid = 148 * 8;
  if (dtype == 0)
    fill_normal_kernel<float><<<grid, 256, 0, st>>>((float*)out, n, key, scale);
  else
    fill_normal_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((__nv_bfloat16*)out, n, key, scale);
  return (int)cudaGetLastError();
}

}  // extern "C"
