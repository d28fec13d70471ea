/*
 * mf.h -- C ABI of the MapFlow hot path on NVIDIA B200 (sm_100a).
 *
 * MapFlow ("Accelerating Cross-Model LLM Inference via Attention Map Reuse",
 * Jin, Luo, Cui, Miao) lets a receiver LLM reuse the attention maps a sender
 * LLM computed on the same context instead of recomputing its own prefill
 * attention.  This library implements the two data-parallel kernels of that
 * method:
 *
 *   mf_compress      block-sparse compression of one sender layer's maps.
 *                    Page "MapFlow开源:大模型换班,Prefill为何能快20%?"
 *                    (aitest123.com), section "存不下、读得慢?三个工程优化手段",
 *                    subsection 1 "只存重要的:块稀疏压缩": the map is cut into
 *                    regular 2-D blocks, block statistics are computed first and
 *                    the important blocks are then chosen by cumulative
 *                    attention probability, without assembling a second dense
 *                    matrix.
 *
 *   mf_map_retrieve  the fused retrieval kernel.  Same page and section,
 *                    subsection 3 "算得省的:融合内核执行": read the sparse blocks,
 *                    form the linear combination of sender heads into receiver
 *                    heads on chip, multiply by the receiver's own V and
 *                    accumulate; layer and head mapping from the section
 *                    "不传 KV Cache,改传注意力关系" ("层映射", "头映射");
 *                    PagedAttention, chunked prefill and varlen packing from the
 *                    closing paragraph of subsection 3.
 *
 * Conventions (all calls):
 *   - The caller owns every buffer.  The library never allocates or frees
 *     device memory; scratch space is passed in as `workspace`.
 *   - Pointers documented "device" are CUDA device (or managed) pointers on
 *     the current device; "host" pointers are read during the call only.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  The call returns after host-side validation and
 *     launch.  Host-detectable errors return a status immediately and enqueue
 *     nothing.
 *   - Errors found on the device (a BSR index out of range, a page id out of
 *     range, nnz above capacity, a pipeline wait that ran out of time) set a
 *     per-device status word and never fault: the kernel skips the offending
 *     access.  mf_get_status() reads and clears it.
 *   - mf_last_error() returns a message for the calling host thread's last
 *     failed call.
 *   - All calls are thread-safe for distinct streams.
 */
#ifndef MF_H
#define MF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MF_OK = 0,
  MF_ERR_INVALID = 1,      /* a descriptor field is out of range or inconsistent */
  MF_ERR_UNSUPPORTED = 2,  /* valid, but a shape this build does not handle */
  MF_ERR_CAPACITY = 3,     /* device: more kept blocks than capacity_blocks */
  MF_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  MF_ERR_TIMEOUT = 5,      /* device: a pipeline wait ran out of time */
  MF_ERR_DEVICE_INDEX = 6  /* device: a BSR row/column or page id was out of range */
} mf_status;

typedef enum { MF_F32 = 0, MF_BF16 = 1 } mf_dtype;

/* ------------------------------------------------------------------------------
 * Compression of one sender layer.
 *
 * For every sequence s of the varlen pack (length L_s = cu_seqlens[s+1] -
 * cu_seqlens[s], nqb_s = ceil(L_s / B) query blocks, Lp_s = nqb_s * B) the dense
 * maps are [h_s][Lp_s][Lp_s] row-major, starting at element map_seq_offset[s] of
 * `maps`.  Only the causal blocks (kb <= qb) are read; entries with j > i, or
 * i or j >= L_s, are ignored and stored as 0.
 *
 * For each query block qb (rows [qb*B, qb*B+B) of each sequence, in pack order):
 *   mass[kb] = sum over sender heads s, rows i, keys j <= i of A_s[i][j], kb <= qb
 *   the diagonal block is kept; the other blocks are taken in (mass desc, kb asc)
 *   order until the running sum S reaches tau * total, where total is the row's
 *   mass summed in that same order (float64).  Kept indices are stored ascending.
 * Output is BSR over all query blocks of the pack:
 *   row_ptr[r], r = 0..R (R = sum_s nqb_s), int32 device, row r = (s, qb) in order
 *   col_idx[n], int32 device, key-block index local to the sequence
 *   values[n][h_s][B][B], map dtype, device: exact copies of the kept blocks
 *   *nnz_out (int32 device) = row_ptr[R]
 * If more than capacity_blocks blocks are kept, the first capacity_blocks are
 * written, *nnz_out holds the true count and the status word reports
 * MF_ERR_CAPACITY.
 * block_mass_out (optional, float64 device) receives every causal block's mass:
 * sequence s, row qb, block kb at cb_base_s + qb*(qb+1)/2 + kb, where cb_base_s =
 * sum over earlier sequences of nqb*(nqb+1)/2.
 * Requirements: B in {32, 64, 128}; 0 <= tau <= 1; map_seq_offset[s] a multiple
 * of 16 bytes; nqb_s <= 4096.
 * ------------------------------------------------------------------------------ */
typedef struct {
  const void* maps;                /* device */
  mf_dtype dtype;                  /* MF_F32 or MF_BF16 (maps and values) */
  const int64_t* map_seq_offset;   /* device [nseq], element offsets */
  const int32_t* cu_seqlens;       /* device [nseq + 1] */
  int32_t nseq;                    /* >= 1 */
  int32_t max_seqlen;              /* host bound: every L_s <= max_seqlen */
  int32_t h_s;                     /* sender heads, 1..256 */
  int32_t B;                       /* block size */
  double tau;                      /* cumulative-mass threshold */
  int32_t* row_ptr;                /* device out [R + 1] */
  int32_t* col_idx;                /* device out [capacity_blocks] */
  void* values;                    /* device out [capacity_blocks][h_s][B][B] */
  int64_t capacity_blocks;
  int32_t* nnz_out;                /* device out [1] */
  double* block_mass_out;          /* device out, optional (NULL) */
} mf_compress_desc;

/* Bytes of scratch `mf_compress` needs for this descriptor (an upper bound computed
 * from nseq, max_seqlen, B and capacity_blocks).  Returns MF_OK or MF_ERR_INVALID. */
mf_status mf_compress_workspace_size(const mf_compress_desc* desc, size_t* bytes);

/* Enqueue compression.  workspace: device, >= mf_compress_workspace_size bytes,
 * 256-byte aligned, not used by any other call until this one completes. */
mf_status mf_compress(const mf_compress_desc* desc, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Compression for callers that cannot allocate device memory.  (This entry point is
 * a property of this library, not of the MapFlow method: the pages have no
 * counterpart.)  Some callers may not call cudaMalloc at all: a plugin inside a host
 * program that owns every byte of device memory through its own pool, or a
 * latency-critical path where an allocation's implicit device synchronisation is
 * not acceptable.  Such a caller passes only the inputs and outputs; the scratch
 * space mf_compress takes as `workspace` comes instead from a file-scope device
 * array of MF_STATIC_WORKSPACE_BYTES that every device loading this library holds
 * until the process exits.  Nothing is allocated or freed by this call.
 *   - The first call on a device looks up the array's device address on the current
 *     device (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - A descriptor whose scratch need (mf_compress_workspace_size) exceeds
 *     MF_STATIC_WORKSPACE_BYTES is rejected with MF_ERR_UNSUPPORTED and a message.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents (each call writes every scratch word before reading it).  Calls whose
 *     work overlaps on the GPU race on it: issue them on one stream, or order them.
 * Outputs and errors are those of mf_compress. */
#define MF_STATIC_WORKSPACE_BYTES (8u << 20)
mf_status mf_compress_static(const mf_compress_desc* desc, void* stream);

/* ------------------------------------------------------------------------------
 * mf_compress_qk: compression straight from the sender's queries and keys, with no
 * dense map anywhere (MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?",
 * section "存不下、读得慢?三个工程优化手段", subsection 1: block statistics are
 * computed first, then the kept blocks, without assembling the dense matrix).
 * The map of sender head s is its causal attention distribution
 *   A_s[i][j] = exp(scale q_{i,s} . k_{j,g}) / sum_{j' <= i} exp(scale q_{i,s} . k_{j',g}),
 * j <= i < L, g = floor(s * h_kv / h_s).  Three passes over the causal key blocks:
 *   1. per (row, key block, head): the block's max scaled score and exp-sum (tensor cores
 *      for q.k), to a scratch buffer;
 *   2. per row: the log-sum-exp; per causal block: the head-summed mass (float64, fixed
 *      order); then selection and row_ptr / col_idx exactly as mf_compress does;
 *   3. the kept blocks only: A recomputed and written as bfloat16 values.
 * Output layout, capacity handling and block_mass_out are those of mf_compress (values
 * bfloat16).  lse_out (optional, float device [h_s][T]) receives each row's log2-sum-exp
 * of the scores scaled by scale * log2(e).
 * Requirements: dtype MF_BF16; d = 128; B = 64; h_s a multiple of h_kv; Q and K
 * 16-byte aligned.  Q: [T][h_s][d], K: [T][h_kv][d] (varlen pack by cu_seqlens, T = total
 * tokens, HOST value), both bfloat16 device.
 * ------------------------------------------------------------------------------ */
typedef struct {
  const void* Q;                   /* device [T][h_s][d] bf16 */
  const void* K;                   /* device [T][h_kv][d] bf16 */
  mf_dtype dtype;                  /* MF_BF16 */
  const int32_t* cu_seqlens;       /* device [nseq + 1] */
  int32_t nseq;                    /* >= 1 */
  int32_t max_seqlen;              /* host bound: every L_s <= max_seqlen */
  int64_t T;                       /* host: total tokens (cu_seqlens[nseq]) */
  int32_t h_s, h_kv, d;            /* sender query heads, key heads, head dim */
  float scale;                     /* softmax scale; 0 means 1 / sqrt(d) */
  int32_t B;                       /* block size (64) */
  double tau;                      /* cumulative-mass threshold */
  int32_t* row_ptr;                /* device out [R + 1] */
  int32_t* col_idx;                /* device out [capacity_blocks] */
  void* values;                    /* device out [capacity_blocks][h_s][B][B] bf16 */
  int64_t capacity_blocks;
  int32_t* nnz_out;                /* device out [1] */
  double* block_mass_out;          /* device out, optional (NULL) */
  float* lse_out;                  /* device out, optional (NULL) [h_s][T] */
} mf_compress_qk_desc;

/* Scratch bytes of mf_compress_qk (an upper bound from nseq, max_seqlen, T, h_s and
 * capacity_blocks; the per-block statistics take h_s * causal blocks * B * 8 bytes). */
mf_status mf_compress_qk_workspace_size(const mf_compress_qk_desc* desc, size_t* bytes);

/* Enqueue compression from Q and K.  workspace as for mf_compress.  Errors: MF_ERR_INVALID
 * for a bad descriptor, MF_ERR_UNSUPPORTED outside the requirements, MF_ERR_CUDA for a
 * launch failure; device-side conditions through mf_get_status. */
mf_status mf_compress_qk(const mf_compress_qk_desc* desc, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ------------------------------------------------------------------------------
 * Fused retrieval for receiver layers l = l_r_begin .. l_r_end-1.
 *
 * Receiver layer l reads sender layer layer_map[l] (a BSR from mf_compress).  For
 * each sequence s of the batch, k_len = cu_seqlens_k[s+1] - cu_seqlens_k[s] is
 * the prefix length and q_len = cu_seqlens_q[s+1] - cu_seqlens_q[s] the number of
 * queries: the queries are the last q_len tokens of the prefix (chunked prefill;
 * q_len = k_len for a whole sequence).  k_len - q_len must be a multiple of B.
 * Query position i of sequence s lives in BSR row qblock_base[s] + i / B.  For
 * every query i and receiver head r (g(r) = r * h_kv / h_r, contiguous GQA groups):
 *   P_r[i][j] = sum_s W[l][r][s] * A_s[i][j]          over kept keys j <= i
 *   O[l'][cu_seqlens_q[s] + (i - (k_len - q_len))][r][:] = sum_j P_r[i][j] * V_l[j][g(r)][:]
 * with l' = l - l_r_begin.  V_l = V + l * v_layer_stride elements:
 *   contiguous: [T_k][h_kv][d], key j of sequence s at token cu_seqlens_k[s] + j;
 *   paged:      [n_pages][page_size][h_kv][d], key j at page
 *               block_table[s * max_pages + j / page_size], row j % page_size.
 * O (dtype v_dtype, or float32 with flag MF_RETRIEVE_O_F32) is
 * [l_r_end - l_r_begin][T_q][h_r][d] with layer stride o_layer_stride elements
 * (0 = T_q * h_r * d).
 * Arithmetic: MF_F32 maps/V run in float32 throughout.  MF_BF16 maps and V run on
 * tcgen05 tensor cores: W is split into a bf16 pair (hi + lo, ~16 bits) and the mixed
 * map P is accumulated in float32.  P.V (float32 accumulation) then takes P either as
 * a bf16 pair (hi truncated, lo the rounded remainder: P to ~16 bits) or rounded once
 * to bf16 (round to nearest even, as a bf16 attention kernel rounds its P): the pair
 * with float32 O (MF_RETRIEVE_O_F32), with flag MF_RETRIEVE_P_SPLIT, and in the first
 * query block of every sequence (rows with at most B keys, where |P| is largest);
 * one rounding elsewhere, which adds at most 2^-8 |P_r[i][j]| |V[j]| per key to the
 * error of O.  A bf16 O is rounded to nearest even.  Each output row's accumulation
 * order depends only on its query block's kept blocks, so chunked, paged and varlen
 * layouts give bit-identical rows.
 * Requirements: h_r % h_kv == 0; layer_map[l] < n_sender_layers; d <= 256.
 * The tensor-core path needs MF_BF16 maps and V (V 16-byte aligned), B in {64, 128},
 * d = 128, h_r / h_kv <= 4, h_s <= 64 and (if paged) page_size in {8, 16, 32, 64};
 * other shapes run a float32 SIMT kernel.
 * ------------------------------------------------------------------------------ */
typedef struct {
  const int32_t* row_ptr;          /* device */
  const int32_t* col_idx;          /* device */
  const void* values;              /* device [capacity_blocks][h_s][B][B] */
  int64_t capacity_blocks;
} mf_bsr;

#define MF_RETRIEVE_FORCE_SIMT 1   /* flags: run the SIMT kernel even where tensor cores apply */
#define MF_RETRIEVE_O_F32 2        /* flags: O is float32 (the unrounded float32 accumulators);
                                      tensor-core path only (bf16 maps and V), else
                                      MF_ERR_UNSUPPORTED */
#define MF_RETRIEVE_P_SPLIT 4      /* flags: P.V takes P as a bf16 pair in every query block
                                      (tensor-core path; the SIMT path is float32 anyway) */

typedef struct {
  const mf_bsr* layers;            /* host [n_sender_layers] */
  int32_t n_sender_layers;
  mf_dtype map_dtype;
  int32_t h_s, B;
  const int32_t* layer_map;        /* host [>= l_r_end] */
  int32_t l_r_begin, l_r_end;
  const float* W;                  /* device [L_r][h_r][h_s] float32, indexed by l */
  const void* V;                   /* device, see above */
  mf_dtype v_dtype;                /* V and O */
  int64_t v_layer_stride;          /* elements; 0 = one V for every layer */
  int32_t paged, page_size, n_pages, max_pages;
  const int32_t* block_table;      /* device [nseq][max_pages] when paged */
  int64_t total_k;                 /* contiguous: rows of V (T_k) */
  const int32_t* cu_seqlens_q;     /* device [nseq + 1] */
  const int32_t* cu_seqlens_k;     /* device [nseq + 1] */
  const int32_t* qblock_base;      /* device [nseq] */
  int32_t nseq, max_seqlen_q;      /* host bound: every q_len <= max_seqlen_q */
  int32_t h_r, h_kv, d;
  void* O;                         /* device out */
  int64_t o_layer_stride;          /* elements */
  int32_t total_q;                 /* T_q */
  int32_t flags;
} mf_retrieve_desc;

mf_status mf_map_retrieve(const mf_retrieve_desc* desc, void* stream);

/* Several receivers of one sender in shared launches (the pages' one-sender, several-
 * receivers workflow, MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?", section
 * "它能做什么:三种典型工作流": one sender's compressed maps serve several receiver models).
 * Same results as calling mf_map_retrieve on descs[0..n-1] in order (bitwise).  When every
 * receiver takes the tensor-core path and all share the sender blocks of every layer step
 * (the same mf_bsr pointers), the query / key packing (cu_seqlens_q/k and qblock_base
 * pointers, nseq, max_seqlen_q) and the number of receiver layers, up to four receivers share
 * each launch: the CTAs of all receivers walk the same query blocks together, so the kept
 * map tiles are read from HBM once per step and reused from L2.  Otherwise the receivers run
 * one after another.  The receivers' O regions must not overlap.  Errors as for
 * mf_map_retrieve (the first failing descriptor). */
mf_status mf_map_retrieve_multi(const mf_retrieve_desc* descs, int n, void* stream);

/* 1 when mf_map_retrieve_multi would share launches among descs, 0 when it would run them
 * one by one, -1 for an invalid descriptor. */
int mf_retrieve_multi_fused(const mf_retrieve_desc* descs, int n);

/* Which kernel mf_map_retrieve would launch: 0 = float32 SIMT, 1 = tcgen05.
 * Returns -1 for an invalid descriptor. */
int mf_retrieve_path(const mf_retrieve_desc* desc);

/* ------------------------------------------------------------------------
 * Head-map calibration (offline).  MapFlow page "MapFlow开源:大模型换班,Prefill为何能快20%?",
 * section "不传 KV Cache,改传“注意力关系”" (head and layer mapping): the weights that map
 * sender heads onto receiver heads are learned once, offline, with both models frozen; the
 * page states no objective.  Reading taken: least squares of
 * every receiver head's map on the sender heads' maps over the causal positions (i < L,
 * j <= i) of the calibration sequences, with an optional ridge term.  The layer map is then
 * chosen by the smallest residual (caller side: one Gram per candidate sender layer).
 *
 * mf_calib_gram adds, for each sequence, the Gram matrix of the stacked features
 * (X_0 .. X_{h_s-1}, Y_0 .. Y_{h_r-1}) over its causal positions into `gram`
 * (device, double [F][F], F = h_s + h_r, row-major, not cleared by the call).
 * Maps are dense, as for mf_compress: sequence s has [h][Lp][Lp] elements
 * (Lp = ceil(L / B) * B) at element offset *_seq_offset[s] (HOST arrays here: the
 * calibration is offline and its launches are planned on the host).  Entries with
 * j > i or in the padding are never used.  bf16 maps with h_s % 8 == 0 and
 * F <= 128 run on tcgen05 tensor cores; other shapes and float32 on a SIMT kernel.
 * Limits: 1 <= h_s <= 64, 1 <= h_r <= 64, B in {32, 64, 128}, L <= 65536.
 * The caller owns every buffer; the workspace (mf_calib_workspace_size bytes,
 * 256-byte aligned) holds per-CTA partial Grams.  Asynchronous on `stream`.
 */
typedef struct {
  const void* sender_maps;              /* device: maps of one sender layer */
  const void* receiver_maps;            /* device: maps of one receiver layer, same dtype */
  mf_dtype dtype;
  const int64_t* sender_seq_offset;     /* HOST [nseq] element offsets into sender_maps */
  const int64_t* receiver_seq_offset;   /* HOST [nseq] element offsets into receiver_maps */
  const int32_t* seqlens;               /* HOST [nseq] sequence lengths L */
  int nseq;
  int h_s, h_r, B;
  double* gram;                         /* device [F][F] double, accumulated into */
} mf_calib_desc;

mf_status mf_calib_workspace_size(const mf_calib_desc* desc, size_t* bytes);
mf_status mf_calib_gram(const mf_calib_desc* desc, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Least-squares head map from an accumulated Gram (device, double [F][F]):
 * W (device, float [h_r][h_s]) solves (G_ss + ridge I) W^T = G_sr by Cholesky in
 * double; residual (device, double [h_r], may be NULL) receives
 * sum (Y_r - W_r . X)^2 over the positions of the Gram.  A sender Gram that is not
 * positive definite (a silent sender head with ridge = 0) sets status bit 32
 * (MF_ERR_INVALID from mf_get_status) and leaves W and residual at 0.
 * Asynchronous on `stream`. */
mf_status mf_calib_solve(const double* gram, int h_s, int h_r, double ridge, float* W,
                         double* residual, void* stream);

/* Which Gram kernel mf_calib_gram launches: 0 = SIMT, 1 = tcgen05; -1 invalid. */
int mf_calib_path(const mf_calib_desc* desc);

/* ------------------------------------------------------------------------------
 * Prefix-hash cache of compressed blocks (MapFlow page "MapFlow开源:大模型换班,Prefill为何
 * 能快20%?", section "存不下、读得慢?三个工程优化手段", subsection 2: the kept blocks are
 * indexed by a prefix hash that carries the preceding context, the receiver finds its blocks
 * through it, and fetching them may overlap the receiver's first layers).
 *
 * mf_prefix_hashes: out[k] (k < ceil(L / B)) = 64-bit FNV-1a of the little-endian bytes of
 * tokens[0 .. min((k + 1) B, L)), i.e. of the whole prefix up to the end of query block k, so
 * equal hashes mean equal preceding context.  Host only.
 *
 * The cache: the caller gives one device buffer (pool, pool_bytes, 16-byte aligned) that the
 * cache cuts into slots of one kept block (h_s * B * B elements of dtype); the index, free list
 * and least-recently-used order live on the host (thread-safe).  An entry is one query-block
 * row of one sender layer, keyed by (layer, prefix hash).
 *   mf_cache_put: copies rows [row0, row0 + nrows) of a compressed layer into the pool (rows
 *     already present only move to the front of the LRU order; rows that do not fit evict the
 *     least recently used rows; a row larger than the pool is skipped, and so is a row that
 *     reaches past bsr->capacity_blocks, whose blocks an overflowed compression did not all
 *     write).  row_ptr_host and
 *     col_idx_host are host copies of the BSR's index arrays.  *inserted (optional) = rows added.
 *   mf_cache_get: assembles the longest cached prefix of a request's rows (hashes[0 .. nrows))
 *     into a BSR: row_ptr [hit + 1], col_idx, values (device, capacity blocks).  *hit (host) =
 *     rows found; the prefix ends at the first miss or where capacity runs out.
 *   Both enqueue copies on `stream` and return at once; a get may run on a side stream while
 *   the receiver computes its first layers (order the retrieval after it with an event).  The
 *   caller orders a put after the gets that precede it (a put may evict and overwrite slots).
 *   mf_cache_stats: rows, used slots, free slots, hits, misses, evictions (int64[6]).
 * ------------------------------------------------------------------------------ */
typedef struct mf_block_cache mf_block_cache;
typedef struct {
  void* pool;          /* device, owned by the caller, alive until mf_cache_destroy */
  size_t pool_bytes;
  int32_t h_s, B;
  mf_dtype dtype;
} mf_cache_desc;

mf_status mf_prefix_hashes(const int32_t* tokens, int64_t L, int32_t B, uint64_t* out);
mf_status mf_cache_create(const mf_cache_desc* desc, mf_block_cache** out);
void mf_cache_destroy(mf_block_cache* cache);
mf_status mf_cache_put(mf_block_cache* cache, int32_t layer, const mf_bsr* bsr,
                       const int32_t* row_ptr_host, const int32_t* col_idx_host, int64_t row0,
                       int32_t nrows, const uint64_t* hashes, int64_t* inserted, void* stream);
mf_status mf_cache_get(mf_block_cache* cache, int32_t layer, const uint64_t* hashes, int32_t nrows,
                       int32_t* row_ptr, int32_t* col_idx, void* values, int64_t capacity_blocks,
                       int32_t* hit, void* stream);
mf_status mf_cache_stats(mf_block_cache* cache, int64_t* out6);

/* ------------------------------------------------------------------------------
 * Bounded waits (a property of this library; the MapFlow pages have no counterpart).
 * Every pipeline wait inside the tensor-core kernels (mf_map_retrieve and
 * mf_map_retrieve_multi on the tcgen05 path, mf_compress_qk, mf_calib_gram on the tcgen05
 * path) gives up after a time limit: the CTA then records MF_ERR_TIMEOUT in the status word,
 * every role of the CTA stops, the copies and MMAs it already issued are waited for (bounded
 * by 2 s) and its tensor memory is released, so the kernel returns and the context stays
 * usable.  mf_set_wait_limit sets that limit, in nanoseconds, for the launches made after the
 * call by any thread of this process; limit_ns = 0 restores the default of 2 s.  With
 * stall != 0 those launches also make the MMA-issuing warp of every CTA first wait on a
 * barrier that nothing arrives at, so the limit is certain to run out: a way to exercise the
 * timeout path without a fault or a hang.  The outputs of a launch that timed out are
 * undefined; a later call with stall = 0 computes normally.  Always returns MF_OK.
 * ------------------------------------------------------------------------------ */
mf_status mf_set_wait_limit(uint64_t limit_ns, int stall);

/* Synchronise `stream`, then read and clear this device's status word.  *bits
 * (optional) receives the raw bits: 1 index out of range, 2 capacity, 4 wait
 * timeout, 8 misaligned input, 16 page id out of range, 32 singular
 * calibration Gram.  Returns MF_OK when no bit was set, else the status of the lowest
 * set bit. */
mf_status mf_get_status(void* stream, uint32_t* bits);

/* Message for the calling thread's last failed call ("" if none). */
const char* mf_last_error(void);

/* Library version string. */
const char* mf_version(void);

/* sizeof of this header's structs as the library was compiled, for bindings that
 * mirror them: which = 0 mf_compress_desc, 1 mf_bsr, 2 mf_retrieve_desc,
 * 3 mf_calib_desc, 4 mf_compress_qk_desc.
 * Returns 0 for any other value. */
size_t mf_abi_struct_size(int which);

#ifdef __cplusplus
}
#endif

#endif /* MF_H */
