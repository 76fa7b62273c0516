// Host-visible part of the short-unit decode kernel (short_decode.cu): its parameters and launcher.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace ta {

constexpr int kShortMaxSeq = 128;       // sequences per launch
constexpr int64_t kShortMaxLen = 2048;  // longest unit the automatic choice sends to this kernel
constexpr int kShortMaxChunks = 64;     // prefix chunks it can fold per row
constexpr int kErrShortWait = 5;        // error word: a bounded wait of this kernel ran out

// One launch: persistent CTAs over the (sequence, KV head) units of up to kShortMaxSeq
// sequences, bf16 q/K/V with head_dim 128.
struct ShortParams {
  const __nv_bfloat16* q;  // [B][Hq][D], this launch's first sequence
  const __nv_bfloat16* k;  // cache bases; kv_off[b] is relative to them
  const __nv_bfloat16* v;
  float* out;              // [B][Hq][D]
  float* lse;              // [B][Hq]
  int* err;                // workspace error word: read for the prefix pass's status, set on a timeout
  // Prefix chunk statistics folded into every row (nullptr: none); same layout as the split
  // kernel's SplitParams::pre_part, already offset to this launch's first sequence.
  const float* pre_part;
  int pre_chunks, pre_rows, pre_stride;
  int n_kv_heads, n_q_heads, n_seq;
  float scale_log2;
  int64_t wait_limit_ns;
  int debug_skip_stage1;  // test hook: 0 off, s > 0: CTA 0 never loads its key stage s - 1
  int64_t kv_off[kShortMaxSeq];   // element offset of sequence b's [Hkv][S_b][D] block
  int64_t seq_len[kShortMaxSeq];
};
static_assert(sizeof(ShortParams) <= 4096, "kernel parameters must fit in 4 KB");

// G = n_q_heads / n_kv_heads in {1, 2, 4, 8}.  At most `max_ctas` CTAs (0: the resident
// maximum on `sms` SMs).  With `after_kernel`, the launch may begin while the preceding kernel
// of the stream still runs (programmatic dependent launch): the kernel waits for that kernel's
// completion before it reads pre_part or err.
cudaError_t launch_short_decode(int G, const ShortParams& p, int sms, int max_ctas, bool after_kernel,
                                cudaStream_t st);

}  // namespace ta
