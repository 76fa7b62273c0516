// Host-visible part of the bifurcated (shared-prefix) tensor-core pass: tile shapes, the
// kernel parameters and the launchers; the kernels are in bifurcated_tc.cu.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace ta {

constexpr int kBifRows = 128;       // rows of one M tile (one TMEM lane each)
constexpr int kBifMT = 2;           // M tiles per CTA: the CTA's 256 rows share every K/V tile
constexpr int kBifKeys = 128;       // keys per tile (N of S, K of P V)
constexpr int kBifD = 128;          // head_dim
constexpr int kBifThreads = 384;    // 12 warps
constexpr int kErrBifWait = 4;
constexpr int kErrBifBadPage = 8;  // same word value as the split kernel's bad-page code
constexpr int kBifPartRow = kBifD + 4;  // floats per partial row: m, l, 2 pad, o[D] (16-byte aligned o)
constexpr int kBifMaxSeq = 128;         // sequences per launch of the several-query-tokens form

struct BifParams {
  const void* q;          // [N][Hq][D] bf16
  float* part;            // [chunks][Hkv * rows_per_head][kBifPartRow]: m (log2), l, -, -, o[D]
  int* err;
  int n_samples;
  int n_q_heads;
  int n_kv_heads;
  int rows_per_head;      // N * G
  int n_chunks;
  int64_t prefix_len;
  float scale_log2;
  int64_t wait_limit_ns;
  // mode 0: shared prefix; grid (row-tile pairs, chunks, KV heads); rows are the samples'
  //   query heads of KV head h, each CTA's two M tiles consume every key tile of its chunk.
  // mode 1: several query tokens per sequence; grid (chunks, KV heads, sequences); a unit's
  //   rows_per_head = G * n_queries rows (token j, head g at row j * G + g, at most 128) see
  //   sequence b's keys of KV head h; the CTA's two softmax slots hold the same rows and take
  //   alternate key tiles; row j * G + g sees the first S_b - n_queries + j + 1 keys.
  int mode;
  int n_queries;
  int64_t kv_row0[kBifMaxSeq];  // mode 1: tensor-map row of key 0 of sequence b, KV head 0
  int64_t kv_len[kBifMaxSeq];   // mode 1: S_b
  // Mode 1 over a paged cache (block_table != nullptr): the tensor maps cover the page pools
  // [num_pages][Hkv][page_size][D] with boxes of min(page_size, 128) rows; sequence b's block i
  // is page block_table[b * bt_stride + i] (the launch group's first sequence's row first).
  const int32_t* block_table;
  int64_t bt_stride;
  int64_t num_pages;
  int log2_page;
  // mode 2: context encoding with anchor blocks (one context of ctx_len tokens); grid (query
  //   tiles, KV heads); query tile qt holds positions qt * n_pos .. (n_pos = 128 / G, G heads
  //   each, row j * G + g); the position at offset o of block i sees the anchor block (keys
  //   [0, block_size), when i > 0) and keys [i * block_size, i * block_size + o]; the tensor maps
  //   cover k, v [Hkv][ctx_len][D].  The CTA merges its two slots and writes out / lse itself.
  int64_t ctx_len;
  int64_t block_size;  // a multiple of kBifKeys
  int n_pos;
  float* out;          // [ctx_len][Hq][D]
  float* lse;          // [ctx_len][Hq]
  // Test hook: 0 off; t + 1: CTA (0, 0, 0) never loads K tile t of its chunk (the products that
  // need it wait until the bounded wait runs out).
  int debug_skip_tile1;
};

// The parameters and the two tensor maps share the 4 KB kernel-parameter space.
static_assert(sizeof(BifParams) + 2 * sizeof(CUtensorMap) <= 4096, "kernel parameters must fit in 4 KB");

// Dynamic shared memory of bif_prefix_kernel (the tile ring plus 1 KB for 1024-byte alignment).
size_t bif_prefix_smem_bytes();

// Raises the kernel's dynamic shared-memory limit on the current device.
cudaError_t bif_prefix_set_smem_limit();

// Prefix pass: grid (M-tile pairs, prefix chunks, KV heads), one CTA per SM.
cudaError_t launch_bif_prefix(dim3 grid, const CUtensorMap& kmap, const CUtensorMap& vmap, const BifParams& p,
                              cudaStream_t st);

// Mode 1: merge of a unit's 2 * n_chunks partials into out [B][n][Hq][D] and lse [B][n][Hq].
cudaError_t launch_merge_chunks(const float* part, int n_chunks, int n_kv_heads, int rows_per_head, int n_queries,
                                float* out, float* lse, int batch, int n_q_heads, const int* err, cudaStream_t st);

}  // namespace ta
