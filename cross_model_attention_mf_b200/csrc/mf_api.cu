// C ABI (include/mf.h): host-side validation, workspace carving, launches, status word.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cstdio>
#include <mutex>
#include <algorithm>
#include <cmath>
#include <string>

#include "mf.h"
#include "mf_internal.cuh"

namespace {

// per-device status word (each device that loads the library has its own copy)
__device__ uint32_t g_status;

thread_local std::string t_err;

mf_status fail(mf_status s, const std::string& msg) {
  t_err = msg;
  return s;
}

uint32_t* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
  return static_cast<uint32_t*>(p);
}

bool is_dtype(int d) { return d == MF_F32 || d == MF_BF16; }

mf_status check_compress(const mf_compress_desc* d) {
  if (!d) return fail(MF_ERR_INVALID, "desc is NULL");
  if (!is_dtype(d->dtype)) return fail(MF_ERR_INVALID, "dtype must be MF_F32 or MF_BF16");
  if (!d->maps || !d->map_seq_offset || !d->cu_seqlens || !d->row_ptr || !d->col_idx ||
      !d->values || !d->nnz_out)
    return fail(MF_ERR_INVALID, "a required pointer is NULL");
  if (d->nseq < 1) return fail(MF_ERR_INVALID, "nseq must be >= 1");
  if (d->max_seqlen < 0) return fail(MF_ERR_INVALID, "max_seqlen must be >= 0");
  if (!(d->B == 32 || d->B == 64 || d->B == 128)) return fail(MF_ERR_INVALID, "B must be 32, 64 or 128");
  if (d->h_s < 1 || d->h_s > 256) return fail(MF_ERR_INVALID, "h_s must be in [1, 256]");
  if (!(d->tau >= 0.0 && d->tau <= 1.0)) return fail(MF_ERR_INVALID, "tau must be in [0, 1]");
  if (d->capacity_blocks < 0) return fail(MF_ERR_INVALID, "capacity_blocks must be >= 0");
  const int64_t nqb = ((int64_t)d->max_seqlen + d->B - 1) / d->B;
  if (nqb > 4096) return fail(MF_ERR_UNSUPPORTED, "more than 4096 query blocks per sequence");
  if ((int64_t)d->nseq * nqb >= (int64_t)1 << 31) return fail(MF_ERR_UNSUPPORTED, "too many rows");
  const int64_t elem = d->dtype == MF_F32 ? 4 : 2;
  if ((int64_t)d->h_s * d->B * d->B * elem * d->capacity_blocks < 0)
    return fail(MF_ERR_INVALID, "capacity overflow");
  if (reinterpret_cast<uintptr_t>(d->maps) % 16 || reinterpret_cast<uintptr_t>(d->values) % 16)
    return fail(MF_ERR_INVALID, "maps and values must be 16-byte aligned");
  return MF_OK;
}

mf_status check_retrieve(const mf_retrieve_desc* d) {
  if (!d) return fail(MF_ERR_INVALID, "desc is NULL");
  if (!is_dtype(d->map_dtype) || !is_dtype(d->v_dtype)) return fail(MF_ERR_INVALID, "bad dtype");
  if (!d->layers || d->n_sender_layers < 1) return fail(MF_ERR_INVALID, "no sender layers");
  if (!d->layer_map) return fail(MF_ERR_INVALID, "layer_map is NULL");
  if (d->l_r_begin < 0 || d->l_r_end < d->l_r_begin) return fail(MF_ERR_INVALID, "bad layer range");
  if (!d->W || !d->V || !d->O || !d->cu_seqlens_q || !d->cu_seqlens_k || !d->qblock_base)
    return fail(MF_ERR_INVALID, "a required pointer is NULL");
  if (d->nseq < 1 || d->max_seqlen_q < 0) return fail(MF_ERR_INVALID, "bad nseq / max_seqlen_q");
  if (d->B < 1 || d->B > 128 || d->h_s < 1 || d->h_s > 256) return fail(MF_ERR_INVALID, "bad B / h_s");
  if (d->h_r < 1 || d->h_kv < 1 || d->h_r % d->h_kv) return fail(MF_ERR_INVALID, "h_r must be a multiple of h_kv");
  if (d->d < 1 || d->d > 256) return fail(MF_ERR_INVALID, "d must be in [1, 256]");
  if (d->paged) {
    if (!d->block_table || d->page_size < 1 || d->n_pages < 1 || d->max_pages < 1)
      return fail(MF_ERR_INVALID, "paged V needs block_table, page_size, n_pages, max_pages");
  } else if (d->total_k < 0) {
    return fail(MF_ERR_INVALID, "total_k must be >= 0");
  }
  for (int l = d->l_r_begin; l < d->l_r_end; ++l) {
    const int ls = d->layer_map[l];
    if (ls < 0 || ls >= d->n_sender_layers) return fail(MF_ERR_INVALID, "layer_map entry out of range");
    const mf_bsr& b = d->layers[ls];
    if (!b.row_ptr || !b.col_idx || !b.values || b.capacity_blocks < 0)
      return fail(MF_ERR_INVALID, "incomplete BSR for a mapped sender layer");
  }
  if (mfi::tc_supported(*d) && reinterpret_cast<uintptr_t>(d->V) % 16)
    return fail(MF_ERR_INVALID, "V must be 16-byte aligned");
  if (d->flags & ~(MF_RETRIEVE_FORCE_SIMT | MF_RETRIEVE_O_F32 | MF_RETRIEVE_P_SPLIT))
    return fail(MF_ERR_INVALID, "unknown retrieve flags");
  if ((d->flags & MF_RETRIEVE_O_F32) && !mfi::tc_supported(*d))
    return fail(MF_ERR_UNSUPPORTED, "float32 O (MF_RETRIEVE_O_F32) needs the tensor-core path");
  if (!mfi::tc_supported(*d) && (int64_t)d->B * d->d > 16384)
    return fail(MF_ERR_UNSUPPORTED, "B * d > 16384 needs the tensor-core path");
  return MF_OK;
}

// Scratch of mf_compress_static: a file-scope device array, so that entry point never
// allocates.  Each device that loads this library holds MF_STATIC_WORKSPACE_BYTES of it
// until the process exits.  In host code `g_static_ws` is only a stand-in for the
// symbol, never a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_static_ws[MF_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices];  // device address of g_static_ws, per device (null: not yet)

// Device address of the static scratch on the current device; looked up once per device.
mf_status static_ws_ptr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(MF_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess || !p)
      return fail(MF_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") + cudaGetErrorString(e));
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return MF_OK;
}

std::atomic<uint64_t> g_wait_ns{0};  // 0: the default limit
std::atomic<int> g_stall{0};

}  // namespace

namespace mfi {
uint64_t wait_limit_ns() {
  const uint64_t v = g_wait_ns.load(std::memory_order_relaxed);
  return v ? v : DRAIN_NS;
}
int wait_stall() { return g_stall.load(std::memory_order_relaxed); }
}  // namespace mfi

namespace {
// receiver layer l of a retrieval descriptor
mfi::RetrieveLayer layer_of(const mf_retrieve_desc& d, int l) {
  const int64_t ve = d.v_dtype == MF_F32 ? 4 : 2;
  const int64_t oe = (d.flags & MF_RETRIEVE_O_F32) ? 4 : ve;
  const int64_t o_stride = d.o_layer_stride ? d.o_layer_stride : (int64_t)d.total_q * d.h_r * d.d;
  const mf_bsr& b = d.layers[d.layer_map[l]];
  mfi::RetrieveLayer L;
  L.row_ptr = b.row_ptr;
  L.col_idx = b.col_idx;
  L.values = b.values;
  L.capacity = b.capacity_blocks;
  L.W = d.W + (int64_t)l * d.h_r * d.h_s;
  L.V = static_cast<const char*>(d.V) + (int64_t)l * d.v_layer_stride * ve;
  L.O = static_cast<char*>(d.O) + (int64_t)(l - d.l_r_begin) * o_stride * oe;
  return L;
}

// receivers that can share launches: all on the tensor-core path, the same sender blocks at
// every layer step, the same query / key packing
bool can_fuse(const mf_retrieve_desc* ds, int n) {
  const mf_retrieve_desc& a = ds[0];
  for (int k = 0; k < n; ++k) {
    const mf_retrieve_desc& b = ds[k];
    if (!mfi::tc_supported(b)) return false;
    if (b.map_dtype != a.map_dtype || b.h_s != a.h_s || b.B != a.B || b.nseq != a.nseq ||
        b.max_seqlen_q != a.max_seqlen_q || b.cu_seqlens_q != a.cu_seqlens_q ||
        b.cu_seqlens_k != a.cu_seqlens_k || b.qblock_base != a.qblock_base ||
        b.l_r_end - b.l_r_begin != a.l_r_end - a.l_r_begin)
      return false;
    for (int j = 0; j < a.l_r_end - a.l_r_begin; ++j) {
      const mf_bsr& x = a.layers[a.layer_map[a.l_r_begin + j]];
      const mf_bsr& y = b.layers[b.layer_map[b.l_r_begin + j]];
      if (x.row_ptr != y.row_ptr || x.col_idx != y.col_idx || x.values != y.values ||
          x.capacity_blocks != y.capacity_blocks)
        return false;
    }
  }
  return true;
}

mf_status check_compress_qk(const mf_compress_qk_desc* d) {
  if (!d) return fail(MF_ERR_INVALID, "desc is NULL");
  if (!d->Q || !d->K || !d->cu_seqlens || !d->row_ptr || !d->nnz_out ||
      (d->capacity_blocks > 0 && (!d->col_idx || !d->values)))
    return fail(MF_ERR_INVALID, "a required pointer is NULL");
  if (d->nseq < 1) return fail(MF_ERR_INVALID, "nseq must be >= 1");
  if (d->max_seqlen < 0 || d->T < 0) return fail(MF_ERR_INVALID, "max_seqlen and T must be >= 0");
  if (d->h_s < 1 || d->h_s > 256 || d->h_kv < 1 || d->h_s % d->h_kv != 0)
    return fail(MF_ERR_INVALID, "h_s must be in [1, 256] and a multiple of h_kv");
  if (!(d->tau >= 0.0 && d->tau <= 1.0)) return fail(MF_ERR_INVALID, "tau must be in [0, 1]");
  if (d->capacity_blocks < 0) return fail(MF_ERR_INVALID, "capacity_blocks must be >= 0");
  if (!(d->scale >= 0.0f) || std::isinf(d->scale)) return fail(MF_ERR_INVALID, "scale must be finite and >= 0");
  if (d->dtype != MF_BF16) return fail(MF_ERR_UNSUPPORTED, "mf_compress_qk takes bfloat16 Q and K");
  if (d->d != 128) return fail(MF_ERR_UNSUPPORTED, "mf_compress_qk needs d = 128");
  if (d->B != 64) return fail(MF_ERR_UNSUPPORTED, "mf_compress_qk needs B = 64");
  if (d->T >= ((int64_t)1 << 31) - 256) return fail(MF_ERR_UNSUPPORTED, "T too large");
  if ((d->max_seqlen + 63) / 64 > 4096) return fail(MF_ERR_UNSUPPORTED, "more than 4096 query blocks per sequence");
  if ((reinterpret_cast<uintptr_t>(d->Q) | reinterpret_cast<uintptr_t>(d->K) |
       reinterpret_cast<uintptr_t>(d->values)) % 16)
    return fail(MF_ERR_INVALID, "Q, K and values must be 16-byte aligned");
  return MF_OK;
}

mf_status check_calib(const mf_calib_desc* d) {
  if (!d) return fail(MF_ERR_INVALID, "desc is NULL");
  if (!is_dtype(d->dtype)) return fail(MF_ERR_INVALID, "dtype must be MF_F32 or MF_BF16");
  if (!d->sender_maps || !d->receiver_maps || !d->sender_seq_offset || !d->receiver_seq_offset ||
      !d->seqlens || !d->gram)
    return fail(MF_ERR_INVALID, "a required pointer is NULL");
  if (d->nseq < 1) return fail(MF_ERR_INVALID, "nseq must be >= 1");
  if (d->h_s < 1 || d->h_s > 64 || d->h_r < 1 || d->h_r > 64)
    return fail(MF_ERR_UNSUPPORTED, "h_s and h_r must lie in [1, 64]");
  if (!(d->B == 32 || d->B == 64 || d->B == 128)) return fail(MF_ERR_INVALID, "B must be 32, 64 or 128");
  if (mfi::calib_path(*d) == 0 && d->h_s + d->h_r > 64)
    return fail(MF_ERR_UNSUPPORTED, "h_s + h_r > 64 needs bf16 maps with h_s % 8 == 0");
  for (int s = 0; s < d->nseq; ++s) {
    if (d->seqlens[s] < 0 || d->seqlens[s] > 65536) return fail(MF_ERR_INVALID, "a sequence length is out of [0, 65536]");
    if (d->sender_seq_offset[s] < 0 || d->receiver_seq_offset[s] < 0)
      return fail(MF_ERR_INVALID, "negative map offset");
    if (d->sender_seq_offset[s] % 8 || d->receiver_seq_offset[s] % 8)
      return fail(MF_ERR_INVALID, "map offsets must be multiples of 8 elements (16-byte aligned rows)");
  }
  if (reinterpret_cast<uintptr_t>(d->sender_maps) % 16 || reinterpret_cast<uintptr_t>(d->receiver_maps) % 16)
    return fail(MF_ERR_INVALID, "maps must be 16-byte aligned");
  return MF_OK;
}
}  // namespace

extern "C" {
#pragma GCC visibility push(default)

const char* mf_version(void) { return "mapflow-b200 0.1.0 (sm_100a)"; }

const char* mf_last_error(void) { return t_err.c_str(); }

size_t mf_abi_struct_size(int which) {
  switch (which) {
    case 0: return sizeof(mf_compress_desc);
    case 1: return sizeof(mf_bsr);
    case 2: return sizeof(mf_retrieve_desc);
    case 3: return sizeof(mf_calib_desc);
    case 4: return sizeof(mf_compress_qk_desc);
    default: return 0;
  }
}

mf_status mf_compress_workspace_size(const mf_compress_desc* desc, size_t* bytes) {
  if (!bytes) return fail(MF_ERR_INVALID, "bytes is NULL");
  if (!desc) return fail(MF_ERR_INVALID, "desc is NULL");
  if (desc->nseq < 1 || desc->max_seqlen < 0 || !(desc->B == 32 || desc->B == 64 || desc->B == 128) ||
      desc->capacity_blocks < 0)
    return fail(MF_ERR_INVALID, "bad nseq / max_seqlen / B / capacity");
  *bytes = mfi::compress_ws_layout(*desc, nullptr, nullptr);
  return MF_OK;
}

mf_status mf_compress(const mf_compress_desc* desc, void* workspace, size_t workspace_bytes,
                      void* stream) {
  mf_status s = check_compress(desc);
  if (s != MF_OK) return s;
  const size_t need = mfi::compress_ws_layout(*desc, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(MF_ERR_INVALID, "workspace missing or smaller than mf_compress_workspace_size");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(MF_ERR_INVALID, "workspace must be 256-byte aligned");
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  mfi::CompressWs ws;
  mfi::compress_ws_layout(*desc, &ws, workspace);
  cudaError_t e = mfi::launch_compress(*desc, ws, st, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("mf_compress launch: ") + cudaGetErrorString(e));
  return MF_OK;
}

mf_status mf_compress_static(const mf_compress_desc* desc, void* stream) {
  mf_status s = check_compress(desc);
  if (s != MF_OK) return s;
  const size_t need = mfi::compress_ws_layout(*desc, nullptr, nullptr);
  if (need > (size_t)MF_STATIC_WORKSPACE_BYTES)
    return fail(MF_ERR_UNSUPPORTED, "mf_compress_static: this descriptor needs " + std::to_string(need) +
                                        " bytes of scratch, more than the static " +
                                        std::to_string((size_t)MF_STATIC_WORKSPACE_BYTES) +
                                        " bytes; use mf_compress with a caller workspace");
  void* ws_ptr = nullptr;
  s = static_ws_ptr(&ws_ptr);
  if (s != MF_OK) return s;
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  // Every scratch word the kernels read is written earlier in the same call, so the
  // contents left by a previous call need no clearing.
  mfi::CompressWs ws;
  mfi::compress_ws_layout(*desc, &ws, ws_ptr);
  cudaError_t e = mfi::launch_compress(*desc, ws, st, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(MF_ERR_CUDA, std::string("mf_compress_static launch: ") + cudaGetErrorString(e));
  return MF_OK;
}

mf_status mf_compress_qk_workspace_size(const mf_compress_qk_desc* desc, size_t* bytes) {
  if (!bytes) return fail(MF_ERR_INVALID, "bytes is NULL");
  mf_status s = check_compress_qk(desc);
  if (s != MF_OK) return s;
  *bytes = mfi::compress_qk_ws_layout(*desc, nullptr, nullptr, nullptr);
  return MF_OK;
}

mf_status mf_compress_qk(const mf_compress_qk_desc* desc, void* workspace, size_t workspace_bytes,
                         void* stream) {
  mf_status s = check_compress_qk(desc);
  if (s != MF_OK) return s;
  const size_t need = mfi::compress_qk_ws_layout(*desc, nullptr, nullptr, nullptr);
  if (!workspace || workspace_bytes < need)
    return fail(MF_ERR_INVALID, "workspace missing or smaller than mf_compress_qk_workspace_size");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(MF_ERR_INVALID, "workspace must be 256-byte aligned");
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  mfi::CompressWs ws;
  mfi::QkWs q;
  mfi::compress_qk_ws_layout(*desc, &ws, &q, workspace);
  std::string err;
  if (!mfi::launch_compress_qk(*desc, ws, q, st, static_cast<cudaStream_t>(stream), &err))
    return fail(MF_ERR_CUDA, "mf_compress_qk: " + err);
  return MF_OK;
}

mf_status mf_prefix_hashes(const int32_t* tokens, int64_t L, int32_t B, uint64_t* out) {
  if ((!tokens && L > 0) || L < 0 || B < 1 || (!out && L > 0)) return fail(MF_ERR_INVALID, "bad tokens / L / B / out");
  uint64_t h = 0xcbf29ce484222325ull;  // FNV-1a 64: offset basis, prime 2^40 + 2^8 + 0xb3
  const int64_t nqb = (L + B - 1) / B;
  for (int64_t k = 0; k < nqb; ++k) {
    const int64_t e = std::min<int64_t>((k + 1) * B, L);
    for (int64_t t = k * B; t < e; ++t) {
      const uint32_t v = (uint32_t)tokens[t];
      for (int b = 0; b < 4; ++b) {
        h ^= (v >> (8 * b)) & 0xFFu;
        h *= 0x100000001b3ull;
      }
    }
    out[k] = h;
  }
  return MF_OK;
}

struct mf_block_cache {
  mfi::BlockCache* c;
  mf_cache_desc d;
};

mf_status mf_cache_create(const mf_cache_desc* desc, mf_block_cache** out) {
  if (!desc || !out) return fail(MF_ERR_INVALID, "desc or out is NULL");
  if (!desc->pool || reinterpret_cast<uintptr_t>(desc->pool) % 16) return fail(MF_ERR_INVALID, "pool must be a 16-byte aligned device pointer");
  if (!is_dtype(desc->dtype) || desc->h_s < 1 || desc->h_s > 256 || !(desc->B == 32 || desc->B == 64 || desc->B == 128))
    return fail(MF_ERR_INVALID, "bad dtype / h_s / B");
  const size_t slot = (size_t)desc->h_s * desc->B * desc->B * (desc->dtype == MF_F32 ? 4 : 2);
  if (desc->pool_bytes < slot) return fail(MF_ERR_INVALID, "pool smaller than one block");
  if (desc->pool_bytes / slot >= ((size_t)1 << 31)) return fail(MF_ERR_UNSUPPORTED, "too many slots");
  *out = new mf_block_cache{mfi::cache_create(*desc), *desc};
  return MF_OK;
}

void mf_cache_destroy(mf_block_cache* cache) {
  if (!cache) return;
  mfi::cache_destroy(cache->c);
  delete cache;
}

mf_status mf_cache_put(mf_block_cache* cache, int32_t layer, const mf_bsr* bsr,
                       const int32_t* row_ptr_host, const int32_t* col_idx_host, int64_t row0,
                       int32_t nrows, const uint64_t* hashes, int64_t* inserted, void* stream) {
  if (!cache || !bsr || !row_ptr_host || !hashes || row0 < 0 || nrows < 0)
    return fail(MF_ERR_INVALID, "bad cache / bsr / row_ptr_host / hashes / rows");
  if (!bsr->values || reinterpret_cast<uintptr_t>(bsr->values) % 16) return fail(MF_ERR_INVALID, "bsr values must be 16-byte aligned");
  for (int32_t r = 0; r < nrows; ++r) {
    const int32_t b0 = row_ptr_host[row0 + r], b1 = row_ptr_host[row0 + r + 1];
    if (b0 < 0 || b1 < b0) return fail(MF_ERR_INVALID, "row_ptr_host is not non-decreasing");
    if (b1 > b0 && !col_idx_host) return fail(MF_ERR_INVALID, "col_idx_host is NULL");
  }
  const int64_t n = mfi::cache_put(cache->c, layer, *bsr, row_ptr_host, col_idx_host, row0, nrows,
                                   hashes, static_cast<cudaStream_t>(stream));
  if (n < 0) return fail(MF_ERR_CUDA, "mf_cache_put: copy launch failed");
  if (inserted) *inserted = n;
  return MF_OK;
}

mf_status mf_cache_get(mf_block_cache* cache, int32_t layer, const uint64_t* hashes, int32_t nrows,
                       int32_t* row_ptr, int32_t* col_idx, void* values, int64_t capacity_blocks,
                       int32_t* hit, void* stream) {
  if (!cache || (!hashes && nrows > 0) || nrows < 0 || !row_ptr || !hit || capacity_blocks < 0 ||
      (capacity_blocks > 0 && (!col_idx || !values)))
    return fail(MF_ERR_INVALID, "bad cache / hashes / outputs");
  if (values && reinterpret_cast<uintptr_t>(values) % 16) return fail(MF_ERR_INVALID, "values must be 16-byte aligned");
  int h = 0;
  if (!mfi::cache_get(cache->c, layer, hashes, nrows, row_ptr, col_idx, values, capacity_blocks, &h,
                      static_cast<cudaStream_t>(stream)))
    return fail(MF_ERR_CUDA, "mf_cache_get: copy launch failed");
  *hit = h;
  return MF_OK;
}

mf_status mf_cache_stats(mf_block_cache* cache, int64_t* out6) {
  if (!cache || !out6) return fail(MF_ERR_INVALID, "cache or out is NULL");
  mfi::cache_stats(cache->c, out6);
  return MF_OK;
}

int mf_retrieve_path(const mf_retrieve_desc* desc) {
  if (check_retrieve(desc) != MF_OK) return -1;
  return mfi::tc_supported(*desc) ? 1 : 0;
}

mf_status mf_map_retrieve(const mf_retrieve_desc* desc, void* stream) {
  mf_status s = check_retrieve(desc);
  if (s != MF_OK) return s;
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  const bool tc = mfi::tc_supported(*desc);
  for (int l = desc->l_r_begin; l < desc->l_r_end; ++l) {
    const mfi::RetrieveLayer L = layer_of(*desc, l);
    if (tc) {
      std::string err;
      // layers after the first start as the previous layer's CTAs exit (different O regions)
      if (!mfi::launch_retrieve_tc(&desc, &L, 1, st, static_cast<cudaStream_t>(stream), &err,
                                   l == desc->l_r_begin))
        return fail(MF_ERR_CUDA, "mf_map_retrieve (tcgen05): " + err);
    } else {
      cudaError_t e = mfi::launch_retrieve_simt(*desc, L, st, static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess)
        return fail(MF_ERR_CUDA, std::string("mf_map_retrieve (simt): ") + cudaGetErrorString(e));
    }
  }
  return MF_OK;
}

int mf_retrieve_multi_fused(const mf_retrieve_desc* descs, int n) {
  if (!descs || n < 1) return -1;
  for (int k = 0; k < n; ++k)
    if (check_retrieve(&descs[k]) != MF_OK) return -1;
  return can_fuse(descs, n) ? 1 : 0;
}

mf_status mf_map_retrieve_multi(const mf_retrieve_desc* descs, int n, void* stream) {
  if (!descs || n < 1) return fail(MF_ERR_INVALID, "descs is NULL or n < 1");
  for (int k = 0; k < n; ++k) {
    mf_status s = check_retrieve(&descs[k]);
    if (s != MF_OK) return s;
  }
  if (!can_fuse(descs, n)) {  // one receiver at a time
    for (int k = 0; k < n; ++k) {
      mf_status s = mf_map_retrieve(&descs[k], stream);
      if (s != MF_OK) return s;
    }
    return MF_OK;
  }
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  const int steps = descs[0].l_r_end - descs[0].l_r_begin;
  for (int j = 0; j < steps; ++j)
    for (int k0 = 0; k0 < n; k0 += 4) {  // up to four receivers share a launch
      const int cnt = n - k0 < 4 ? n - k0 : 4;
      const mf_retrieve_desc* ptrs[4];
      mfi::RetrieveLayer Ls[4];
      for (int k = 0; k < cnt; ++k) {
        ptrs[k] = &descs[k0 + k];
        Ls[k] = layer_of(descs[k0 + k], descs[k0 + k].l_r_begin + j);
      }
      std::string err;
      // launches after the first write other receivers' or layers' O
      if (!mfi::launch_retrieve_tc(ptrs, Ls, cnt, st, static_cast<cudaStream_t>(stream), &err,
                                   j == 0 && k0 == 0))
        return fail(MF_ERR_CUDA, "mf_map_retrieve_multi (tcgen05): " + err);
    }
  return MF_OK;
}

mf_status mf_calib_workspace_size(const mf_calib_desc* desc, size_t* bytes) {
  if (!bytes) return fail(MF_ERR_INVALID, "bytes is NULL");
  mf_status s = check_calib(desc);
  if (s != MF_OK) return s;
  *bytes = mfi::calib_ws_bytes(*desc);
  return MF_OK;
}

int mf_calib_path(const mf_calib_desc* desc) {
  if (check_calib(desc) != MF_OK) return -1;
  return mfi::calib_path(*desc);
}

mf_status mf_calib_gram(const mf_calib_desc* desc, void* workspace, size_t workspace_bytes,
                        void* stream) {
  mf_status s = check_calib(desc);
  if (s != MF_OK) return s;
  if (!workspace || workspace_bytes < mfi::calib_ws_bytes(*desc))
    return fail(MF_ERR_INVALID, "workspace missing or smaller than mf_calib_workspace_size");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(MF_ERR_INVALID, "workspace must be 256-byte aligned");
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  std::string err;
  if (!mfi::launch_calib_gram(*desc, workspace, st, static_cast<cudaStream_t>(stream), &err))
    return fail(MF_ERR_CUDA, err);
  return MF_OK;
}

mf_status mf_calib_solve(const double* gram, int h_s, int h_r, double ridge, float* W,
                         double* residual, void* stream) {
  if (!gram || !W) return fail(MF_ERR_INVALID, "gram and W are required");
  if (h_s < 1 || h_s > 64 || h_r < 1 || h_r > 64) return fail(MF_ERR_UNSUPPORTED, "h_s and h_r must lie in [1, 64]");
  if (!(ridge >= 0.0)) return fail(MF_ERR_INVALID, "ridge must be >= 0");
  uint32_t* st = status_ptr();
  if (!st) return fail(MF_ERR_CUDA, "cannot resolve the device status word");
  cudaError_t e = mfi::launch_calib_solve(gram, h_s, h_r, ridge, W, residual, st,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("calib solve launch: ") + cudaGetErrorString(e));
  return MF_OK;
}

mf_status mf_set_wait_limit(uint64_t limit_ns, int stall) {
  g_wait_ns.store(limit_ns, std::memory_order_relaxed);
  g_stall.store(stall ? 1 : 0, std::memory_order_relaxed);
  return MF_OK;
}

mf_status mf_get_status(void* stream, uint32_t* bits) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("stream: ") + cudaGetErrorString(e));
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof v);
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("status read: ") + cudaGetErrorString(e));
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_status, &zero, sizeof zero);
  if (e != cudaSuccess) return fail(MF_ERR_CUDA, std::string("status clear: ") + cudaGetErrorString(e));
  if (bits) *bits = v;
  if (v == 0) return MF_OK;
  if (v & mfi::ST_INDEX) return fail(MF_ERR_DEVICE_INDEX, "device: BSR index out of range");
  if (v & mfi::ST_CAPACITY) return fail(MF_ERR_CAPACITY, "device: kept blocks exceed capacity");
  if (v & mfi::ST_TIMEOUT) return fail(MF_ERR_TIMEOUT, "device: pipeline wait timed out");
  if (v & mfi::ST_ALIGN) return fail(MF_ERR_INVALID, "device: misaligned map offset");
  if (v & mfi::ST_PAGE) return fail(MF_ERR_DEVICE_INDEX, "device: page id out of range");
  return fail(MF_ERR_INVALID, "device: calibration Gram is not positive definite");
}

}  // extern "C"
