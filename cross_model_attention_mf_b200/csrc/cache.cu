// Prefix-hash cache of compressed blocks, with assembly of a request's BSR on any stream.
//
// MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?" (aitest123.com), section
// "存不下、读得慢?三个工程优化手段", subsection 2 "找得快的:基于前缀哈希的缓存管理": the
// kept blocks differ in number per layer and position, so they are indexed by a prefix hash that
// carries the preceding context; a receiver finds its blocks through that index, and fetching
// them can run in the background while the receiver recomputes its first layers.
//
// Layout.  The caller gives one device buffer; it is cut into slots of one kept block
// (h_s * B * B elements).  A cached entry is one query-block row of one sender layer, keyed by
// (layer, prefix hash of the row's query block): its kept key-block indices (host) and the slots
// holding their values.  The index, the free list and the LRU order live on the host; only the
// block copies run on the GPU.
//
// Copies.  k_cache_copy moves whole blocks (16-byte vector loads, each block split over 8 CTAs);
// the list of (source block, destination block, column) triples, and for a get the row
// pointers, travel as a kernel parameter (in structs of 64, 256 or 1024 entries), so a put or a
// get needs no staging buffer and no synchronisation: it is ordered on the caller's stream like
// any other launch.  Rows evicted by a put may still be read
// by an earlier get on another stream; the caller orders puts after the gets that precede them.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "mf_internal.cuh"

namespace mfi {
namespace {

// A launch carries its copy list as a kernel parameter: (source block, destination block,
// column) triples and, for a get, the row pointers of the assembled rows.  The parameter
// struct comes in three sizes so that a small request does not ship 12 KB of parameters.
template <int N>
struct CopyChunk {
  const uint4* src;   // block k of the source at src + src_blk[k] * blk_vecs
  uint4* dst;
  int32_t* col_dst;   // when not NULL: col_dst[dst_blk[k]] = col[k]
  int32_t* row_ptr;   // when not NULL: row_ptr[rp_first + k] = rp[k], k < rp_n
  int64_t blk_vecs;   // 16-byte vectors per block
  int n, rp_first, rp_n;
  int32_t src_blk[N];
  int32_t dst_blk[N];
  int32_t col[N];
  int32_t rp[N + 1];
};
constexpr int CHUNK_MAX = 1024;  // copies per launch (the largest parameter struct, 16 KB)

// grid (blocks, SPLIT): CTA (k, part) copies part `part` of block k, four 16-byte vectors in
// flight per thread; CTA (0, 0) also writes the row pointers the launch carries
constexpr int SPLIT = 8;
template <int N>
__global__ void __launch_bounds__(256) k_cache_copy(const __grid_constant__ CopyChunk<N> c) {
  const int k = blockIdx.x;
  if (c.row_ptr && k == 0 && blockIdx.y == 0)
    for (int e = threadIdx.x; e < c.rp_n; e += 256) c.row_ptr[c.rp_first + e] = c.rp[e];
  if (k >= c.n) return;
  const uint4* s = c.src + (int64_t)c.src_blk[k] * c.blk_vecs;
  uint4* d = c.dst + (int64_t)c.dst_blk[k] * c.blk_vecs;
  const int64_t per = (c.blk_vecs + SPLIT - 1) / SPLIT;
  const int64_t v0 = per * blockIdx.y, v1 = min(c.blk_vecs, v0 + per);
  for (int64_t v = v0 + threadIdx.x; v < v1; v += 4 * 256) {
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v + u * 256 < v1) r[u] = __ldg(s + v + u * 256);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (v + u * 256 < v1) d[v + u * 256] = r[u];
  }
  if (c.col_dst && blockIdx.y == 0 && threadIdx.x == 0) c.col_dst[c.dst_blk[k]] = c.col[k];
}

struct Key {
  int layer;
  uint64_t hash;
  bool operator==(const Key& o) const { return layer == o.layer && hash == o.hash; }
};
struct KeyHash {
  size_t operator()(const Key& k) const { return (size_t)(k.hash ^ ((uint64_t)k.layer * 0x9E3779B97F4A7C15ull)); }
};
struct Entry {
  std::vector<int32_t> cols;   // kept key blocks, ascending
  std::vector<int32_t> slots;  // pool slot of each
  std::list<Key>::iterator lru;
};

}  // namespace

struct BlockCache {
  std::mutex mu;
  char* pool;
  int64_t slot_bytes, n_slots;
  int h_s, B;
  mf_dtype dtype;
  std::vector<int32_t> free_slots;
  std::unordered_map<Key, Entry, KeyHash> index;
  std::list<Key> lru;  // front = most recently used
  int64_t hits = 0, misses = 0, evicted = 0;
};

namespace {

template <int N>
bool launch_chunk(const char* src, char* dst, int32_t* col_dst, int64_t blk_bytes,
                  const std::vector<int32_t>& s, const std::vector<int32_t>& d,
                  const std::vector<int32_t>& col, size_t k0, int n, int32_t* row_ptr,
                  const std::vector<int32_t>& rp, size_t r0, int rp_n, cudaStream_t st) {
  CopyChunk<N> c;
  c.src = reinterpret_cast<const uint4*>(src);
  c.dst = reinterpret_cast<uint4*>(dst);
  c.col_dst = col_dst;
  c.row_ptr = rp_n > 0 ? row_ptr : nullptr;
  c.blk_vecs = blk_bytes / 16;
  c.n = n;
  c.rp_first = (int)r0;
  c.rp_n = rp_n;
  for (int k = 0; k < n; ++k) {
    c.src_blk[k] = s[k0 + k];
    c.dst_blk[k] = d[k0 + k];
    c.col[k] = col.empty() ? 0 : col[k0 + k];
  }
  for (int k = 0; k < rp_n; ++k) c.rp[k] = rp[r0 + k];
  k_cache_copy<N><<<dim3((unsigned)std::max(n, 1), SPLIT), 256, 0, st>>>(c);
  return cudaGetLastError() == cudaSuccess;
}

// Copies block s[k] of src to block d[k] of dst (and col[k] to col_dst[d[k]] when col_dst is
// set), and writes rp[] to row_ptr[] when row_ptr is set, in as few launches as the parameter
// limit allows.
bool launch_copies(const char* src, char* dst, int32_t* col_dst, int64_t blk_bytes,
                   const std::vector<int32_t>& s, const std::vector<int32_t>& d,
                   const std::vector<int32_t>& col, int32_t* row_ptr,
                   const std::vector<int32_t>& rp, cudaStream_t st) {
  size_t k0 = 0, r0 = 0;
  const size_t n_rp = row_ptr ? rp.size() : 0;
  while (k0 < s.size() || r0 < n_rp) {
    const size_t left = std::max(s.size() - k0, n_rp - r0 > 0 ? n_rp - r0 - 1 : 0);
    const int N = left <= 64 ? 64 : left <= 256 ? 256 : CHUNK_MAX;
    const int n = (int)std::min<size_t>(N, s.size() - k0);
    const int rp_n = (int)std::min<size_t>(N + 1, n_rp - r0);
    bool ok = N == 64 ? launch_chunk<64>(src, dst, col_dst, blk_bytes, s, d, col, k0, n, row_ptr, rp, r0, rp_n, st)
            : N == 256 ? launch_chunk<256>(src, dst, col_dst, blk_bytes, s, d, col, k0, n, row_ptr, rp, r0, rp_n, st)
                       : launch_chunk<CHUNK_MAX>(src, dst, col_dst, blk_bytes, s, d, col, k0, n, row_ptr, rp, r0, rp_n, st);
    if (!ok) return false;
    k0 += n;
    r0 += rp_n;
  }
  return true;
}

}  // namespace

// ------------------------------------------------------------------ host API (called by mf_api)
BlockCache* cache_create(const mf_cache_desc& d) {
  BlockCache* c = new BlockCache();
  c->pool = static_cast<char*>(d.pool);
  c->h_s = d.h_s;
  c->B = d.B;
  c->dtype = d.dtype;
  c->slot_bytes = (int64_t)d.h_s * d.B * d.B * (d.dtype == MF_F32 ? 4 : 2);
  c->n_slots = (int64_t)(d.pool_bytes / (size_t)c->slot_bytes);
  c->free_slots.reserve((size_t)c->n_slots);
  for (int64_t k = c->n_slots - 1; k >= 0; --k) c->free_slots.push_back((int32_t)k);
  return c;
}

void cache_destroy(BlockCache* c) { delete c; }

// Inserts rows [row0, row0 + nrows) of a compressed layer (row_ptr on the host).  Rows already
// cached are refreshed in the LRU order only; a row larger than the whole pool, or one that
// reaches past the BSR's capacity (incomplete), is skipped.
// Returns the number of rows inserted, or -1 on a launch failure.
int64_t cache_put(BlockCache* c, int layer, const mf_bsr& bsr, const int32_t* row_ptr_host,
                  const int32_t* col_idx_host, int64_t row0, int nrows, const uint64_t* hashes,
                  cudaStream_t st) {
  std::lock_guard<std::mutex> g(c->mu);
  std::vector<int32_t> src, dst;
  int64_t inserted = 0;
  for (int r = 0; r < nrows; ++r) {
    const Key key{layer, hashes[r]};
    auto it = c->index.find(key);
    if (it != c->index.end()) {
      c->lru.splice(c->lru.begin(), c->lru, it->second.lru);
      continue;
    }
    const int32_t b0 = row_ptr_host[row0 + r], b1 = row_ptr_host[row0 + r + 1];
    // a row that runs past the BSR's capacity (a compression that overflowed) lost some of its
    // kept blocks: caching it would hand a short row to every later request with this prefix
    if (b1 > bsr.capacity_blocks) continue;
    const int64_t need = (int64_t)b1 - b0;
    if (need <= 0 || need > c->n_slots) continue;
    if ((int64_t)c->free_slots.size() < need && !src.empty()) {
      // a slot freed below may be the target of a copy gathered earlier in this call: launch
      // those copies first, so that stream order puts the new row's copy after them
      if (!launch_copies(static_cast<const char*>(bsr.values), c->pool, nullptr, c->slot_bytes, src,
                         dst, {}, nullptr, {}, st))
        return -1;
      src.clear();
      dst.clear();
    }
    while ((int64_t)c->free_slots.size() < need && !c->lru.empty()) {  // evict the LRU rows
      const Key victim = c->lru.back();
      c->lru.pop_back();
      auto v = c->index.find(victim);
      for (int32_t sl : v->second.slots) c->free_slots.push_back(sl);
      c->index.erase(v);
      ++c->evicted;
    }
    Entry e;
    for (int64_t k = 0; k < need; ++k) {
      const int32_t sl = c->free_slots.back();
      c->free_slots.pop_back();
      e.slots.push_back(sl);
      e.cols.push_back(col_idx_host[b0 + k]);
      src.push_back((int32_t)(b0 + k));
      dst.push_back(sl);
    }
    c->lru.push_front(key);
    e.lru = c->lru.begin();
    c->index.emplace(key, std::move(e));
    ++inserted;
  }
  if (!src.empty() && !launch_copies(static_cast<const char*>(bsr.values), c->pool, nullptr,
                                     c->slot_bytes, src, dst, {}, nullptr, {}, st))
    return -1;
  return inserted;
}

// Assembles the longest cached prefix of a request's query-block rows into a BSR: row_ptr
// [hit + 1], col_idx and values.  *hit receives the number of rows found (the prefix stops at the
// first miss, or where capacity runs out).
bool cache_get(BlockCache* c, int layer, const uint64_t* hashes, int nrows, int32_t* row_ptr,
               int32_t* col_idx, void* values, int64_t capacity, int* hit, cudaStream_t st) {
  std::lock_guard<std::mutex> g(c->mu);
  std::vector<int32_t> src, dst, col, rp{0};
  src.reserve(256); dst.reserve(256); col.reserve(256); rp.reserve((size_t)nrows + 1);
  int h = 0;
  for (int r = 0; r < nrows; ++r) {
    auto it = c->index.find(Key{layer, hashes[r]});
    if (it == c->index.end()) { ++c->misses; break; }
    const Entry& e = it->second;
    if ((int64_t)rp.back() + (int64_t)e.slots.size() > capacity) break;
    for (size_t k = 0; k < e.slots.size(); ++k) {
      src.push_back(e.slots[k]);
      dst.push_back(rp.back() + (int32_t)k);
      col.push_back(e.cols[k]);
    }
    rp.push_back(rp.back() + (int32_t)e.slots.size());
    c->lru.splice(c->lru.begin(), c->lru, it->second.lru);
    ++c->hits;
    ++h;
  }
  *hit = h;
  // one launch (for requests of up to 1024 blocks) copies the blocks and writes row_ptr
  return launch_copies(c->pool, static_cast<char*>(values), col_idx, c->slot_bytes, src, dst, col,
                       row_ptr, rp, st);
}

void cache_stats(BlockCache* c, int64_t* out6) {
  std::lock_guard<std::mutex> g(c->mu);
  out6[0] = (int64_t)c->index.size();
  out6[1] = c->n_slots - (int64_t)c->free_slots.size();
  out6[2] = (int64_t)c->free_slots.size();
  out6[3] = c->hits;
  out6[4] = c->misses;
  out6[5] = c->evicted;
}

}  // namespace mfi
