// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "mf.h"

namespace mfi {

// bits of the per-device status word
enum : uint32_t {
  ST_INDEX = 1u,     // BSR row/column index out of range
  ST_CAPACITY = 2u,  // more kept blocks than capacity
  ST_TIMEOUT = 4u,   // a pipeline wait gave up
  ST_ALIGN = 8u,     // a sequence's map offset is not 16-byte aligned
  ST_PAGE = 16u,     // a page id out of range
  ST_SINGULAR = 32u, // a calibration Gram that is not positive definite
};

// limit of every pipeline wait in the tensor-core kernels (ns) and the test stall flag, as set
// by mf_set_wait_limit (read at each launch)
uint64_t wait_limit_ns();
int wait_stall();
constexpr uint64_t DRAIN_NS = 2000000000ull;  // bound of the waits for work already issued

// scratch of mf_compress (carved out of the caller's workspace)
struct CompressWs {
  int64_t* meta;      // [4 + 4 * nseq]: total rows, total causal blocks, selection ticket, -,
                      // then per sequence (L, nqb, row_base, cb_base)
  double* mass;       // [max_cb] head-summed block masses
  unsigned long long* flags;  // [max_rows] selection look-back: count or prefix per row
  int32_t* kept_row;  // [capacity] BSR row of each kept block
  int64_t max_cb, max_rows;
};

// Computes the layout; with base == nullptr only the size is returned.
size_t compress_ws_layout(const mf_compress_desc& d, CompressWs* ws, void* base);

cudaError_t launch_compress(const mf_compress_desc& d, const CompressWs& ws, uint32_t* status,
                            cudaStream_t st);

// the geometry pass of compression (per-sequence meta; off may be NULL: no map offsets)
cudaError_t launch_meta(const int32_t* cu, const int64_t* off, int nseq, int max_seqlen, int B,
                        int elem_bytes, const CompressWs& ws, uint32_t* status, int32_t* row_ptr,
                        int32_t* nnz_out, cudaStream_t st);
// selection and BSR index build from the masses of every causal block
cudaError_t launch_select(const CompressWs& ws, int nseq, int max_seqlen, int B, const double* mass,
                          double tau, int32_t* row_ptr, int32_t* col_idx, int32_t* nnz_out,
                          int64_t capacity, uint32_t* status, cudaStream_t st);

// scratch of mf_compress_qk beyond CompressWs
struct QkWs {
  float2* ml;         // [h_s][cb_stride][B] per-block max and exp-sum of each row
  float* lse2;        // [h_s][T] row log2-sum-exp
  int64_t cb_stride;  // causal-block capacity of the pack
};
size_t compress_qk_ws_layout(const mf_compress_qk_desc& d, CompressWs* ws, QkWs* q, void* base);
bool launch_compress_qk(const mf_compress_qk_desc& d, const CompressWs& ws, const QkWs& q,
                        uint32_t* status, cudaStream_t st, std::string* err);

// one receiver layer's pointers
struct RetrieveLayer {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const void* values;
  int64_t capacity;
  const float* W;  // [h_r][h_s] of this layer
  const void* V;   // this layer's V
  void* O;         // this layer's O
};

cudaError_t launch_retrieve_simt(const mf_retrieve_desc& d, const RetrieveLayer& l,
                                 uint32_t* status, cudaStream_t st);

bool tc_supported(const mf_retrieve_desc& d);

// one launch for n (1..4) receivers that share the sender BSR layer and the query / key
// packing; returns false and fills *err on a host-side failure (tensor-map encoding, launch).
// Every launch may start while the previous kernel on the stream still runs (programmatic
// dependent launch).  first: the call's first launch, which waits for that kernel before its
// first global access; later launches of one call read nothing the earlier ones write.
bool launch_retrieve_tc(const mf_retrieve_desc* const* ds, const RetrieveLayer* ls, int n,
                        uint32_t* status, cudaStream_t st, std::string* err, bool first = true);

// prefix-hash block cache
struct BlockCache;
BlockCache* cache_create(const mf_cache_desc& d);
void cache_destroy(BlockCache* c);
int64_t cache_put(BlockCache* c, int layer, const mf_bsr& bsr, const int32_t* row_ptr_host,
                  const int32_t* col_idx_host, int64_t row0, int nrows, const uint64_t* hashes,
                  cudaStream_t st);
bool cache_get(BlockCache* c, int layer, const uint64_t* hashes, int nrows, int32_t* row_ptr,
               int32_t* col_idx, void* values, int64_t capacity, int* hit, cudaStream_t st);
void cache_stats(BlockCache* c, int64_t* out6);

// head-map calibration
size_t calib_ws_bytes(const mf_calib_desc& d);
int calib_path(const mf_calib_desc& d);
// returns false and fills *err on a host-side failure
bool launch_calib_gram(const mf_calib_desc& d, void* ws, uint32_t* status, cudaStream_t st,
                       std::string* err);
cudaError_t launch_calib_solve(const double* gram, int h_s, int h_r, double ridge, float* W,
                               double* residual, uint32_t* status, cudaStream_t st);

}  // namespace mfi
