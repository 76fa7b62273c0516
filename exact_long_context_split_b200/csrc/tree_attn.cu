// C ABI of the split decode-attention library (declared in include/tree_attn.h):
// argument checks, the work plan, workspace layout and kernel launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tree_attn.h"
#include "bifurcated_tc.h"
#include "short_decode.h"
#include "split_kv_instances.h"

namespace ta {
namespace {

thread_local int32_t g_last_cuda_error = 0;

// Profiling hook (tree_attn_profile_events): events recorded on the call's stream around the
// launches of the call's main kernel.
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;

struct ProfileSpan {
  cudaStream_t st;
  bool open = false;
  explicit ProfileSpan(cudaStream_t s) : st(s) {}
  void begin() {
    if (g_prof_start && !open) cudaEventRecord(g_prof_start, st);
    open = true;
  }
  void end() {
    if (g_prof_stop) cudaEventRecord(g_prof_stop, st);
  }
};

constexpr size_t kAlign = 256;
constexpr size_t kHeaderBytes = 256;  // error word and spare
constexpr int64_t kDefaultWaitUs = 2000000;
constexpr int64_t kMinTilesPerCta = 2;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

ta_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int32_t>(e);
  return TA_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------
// Kernel instances
// ------------------------------------------------------------------------------------------

template <class V, bool PAGED>
bool pick_variant(ta_dtype dt, int D, int G, KernelInfo* ki) {
  if (dt == TA_BF16) {
    if (D == 64) return split_instance<__nv_bfloat16, V, 64, PAGED>(G, ki);
    if (D == 128) return split_instance<__nv_bfloat16, V, 128, PAGED>(G, ki);
  } else if (dt == TA_F32) {
    if (D == 64) return split_instance<float, V, 64, PAGED>(G, ki);
    if (D == 128) return split_instance<float, V, 128, PAGED>(G, ki);
  }
  return false;
}

bool pick_kernel(ta_dtype dt, int D, int G, bool short_tiles, KernelInfo* ki, bool paged = false) {
  if (paged)
    return short_tiles ? pick_variant<ShortTiles, true>(dt, D, G, ki) : pick_variant<LongTiles, true>(dt, D, G, ki);
  return short_tiles ? pick_variant<ShortTiles, false>(dt, D, G, ki) : pick_variant<LongTiles, false>(dt, D, G, ki);
}

// Tile configuration for a batch: short tiles when the mean (sequence, KV head) unit is
// shorter than 1024 tokens, unless the options force one.
bool use_short_tiles(const int64_t* seqlens, int batch, const ta_options* opts) {
  if (opts && opts->split_tiles == 1) return false;
  if (opts && opts->split_tiles == 2) return true;  // (3, the short-unit kernel, only reaches suffix passes)
  int64_t total = 0;
  for (int b = 0; b < batch; ++b) total += seqlens[b];
  return batch > 0 && total < 1024LL * batch;
}

// Resident CTAs of an instance on the current device (sets the shared-memory opt-in once).
ta_status resident_ctas(const KernelInfo& ki, int* device_out, int* slots_out) {
  static std::mutex mu;
  struct Entry {
    int device;
    void (*fn)(SplitParams);
    int slots;
  };
  static std::vector<Entry> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(mu);
  for (const Entry& c : cache)
    if (c.device == dev && c.fn == ki.fn) {
      *device_out = dev;
      *slots_out = c.slots;
      return TA_OK;
    }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(ki.fn), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(ki.smem));
  if (e != cudaSuccess) return cuda_fail(e);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, reinterpret_cast<const void*>(ki.fn), ki.threads,
                                                    ki.smem);
  if (e != cudaSuccess) return cuda_fail(e);
  if (per_sm < 1) return cuda_fail(cudaErrorInvalidConfiguration);
  cache.push_back(Entry{dev, ki.fn, sms * per_sm});
  *device_out = dev;
  *slots_out = sms * per_sm;
  return TA_OK;
}

// ------------------------------------------------------------------------------------------
// Work plan
// ------------------------------------------------------------------------------------------

struct Group {
  int b0 = 0, nb = 0;
  int P = 0;
  bool unit_aligned = false;
  int64_t NT = 0;
  size_t tickets_off = 0, part_off = 0;  // byte offsets inside the workspace body
  int64_t kv_off[kMaxSeqPerLaunch];
  int64_t len[kMaxSeqPerLaunch];
  int64_t tile_off[kMaxSeqPerLaunch + 1];
  int32_t n_tiles[kMaxSeqPerLaunch];
};

struct Plan {
  std::vector<Group> groups;
  size_t body_bytes = 0;
};

// kv_offsets == nullptr: sequences packed back to back ([Hkv][S_b][D] blocks).
// Otherwise: explicit element offset of each sequence's block (blocks may alias).
ta_status build_plan(const int64_t* seqlens, const int64_t* kv_offsets, int batch, int Hkv, int G, int D,
                     int tile, int slots, const ta_options* opts, Plan* plan) {
  plan->groups.clear();
  size_t body = 0;
  int64_t packed = 0;
  for (int b0 = 0; b0 < batch; b0 += kMaxSeqPerLaunch) {
    Group g;
    g.b0 = b0;
    g.nb = std::min(kMaxSeqPerLaunch, batch - b0);
    int64_t NT = 0;
    for (int i = 0; i < g.nb; ++i) {
      const int64_t S = seqlens[b0 + i];
      g.len[i] = S;
      g.kv_off[i] = kv_offsets ? kv_offsets[b0 + i] : packed;
      packed += S * Hkv * static_cast<int64_t>(D);
      g.n_tiles[i] = static_cast<int32_t>(std::max<int64_t>(1, (S + tile - 1) / tile));
      g.tile_off[i] = NT;
      NT += static_cast<int64_t>(Hkv) * g.n_tiles[i];
    }
    g.tile_off[g.nb] = NT;
    g.NT = NT;
    // Default grid: one CTA per resident slot, but at least kMinTilesPerCta tiles each, so a
    // small problem is not spread into one-tile CTAs whose partial writes and merge tree cost
    // more than their loads (tiny, 22 tiles: 17 us with 8-16 CTAs against 26 us with 22).
    int64_t P = (opts && opts->num_ctas > 0) ? opts->num_ctas
                                             : std::min<int64_t>(slots, std::max<int64_t>(1, NT / kMinTilesPerCta));
    P = std::max<int64_t>(1, std::min<int64_t>(P, NT));
    g.P = static_cast<int>(P);
    const int64_t units = static_cast<int64_t>(g.nb) * Hkv;
    // Many short units: keep each unit in one CTA (no partials, tickets or merge tails) when
    // every unit is at most half a CTA's share of tiles, so the ranges stay balanced.
    int32_t max_unit_tiles = 0;
    for (int i = 0; i < g.nb; ++i) max_unit_tiles = std::max(max_unit_tiles, g.n_tiles[i]);
    g.unit_aligned = units >= P && 2 * static_cast<int64_t>(max_unit_tiles) * P <= NT;
    g.tickets_off = body;
    body = align_up(body + sizeof(int) * units, kAlign);
    g.part_off = body;
    body = align_up(body + sizeof(float) * static_cast<size_t>(P + units) * G * (D + 2), kAlign);
    plan->groups.push_back(g);
  }
  plan->body_bytes = body;
  return TA_OK;
}

// ------------------------------------------------------------------------------------------
// Argument checks
// ------------------------------------------------------------------------------------------

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ta_status check_opts(const ta_options* o) {
  if (!o) return TA_OK;
  if (o->num_ctas < 0 || o->wait_limit_us < 0 || o->debug_skip_tile < -1 || o->debug_skip_stage < 0)
    return TA_ERR_INVALID_ARG;
  if (o->prefix_path < 0 || o->prefix_path > 2) return TA_ERR_INVALID_ARG;
  if (o->split_tiles < 0 || o->split_tiles > 3) return TA_ERR_INVALID_ARG;
  for (int i = 0; i < 2; ++i)
    if (o->reserved[i] != 0) return TA_ERR_INVALID_ARG;
  return TA_OK;
}

ta_status check_shape(const int64_t* seqlens, int batch, int Hq, int Hkv, int D, ta_dtype dt, KernelInfo* ki) {
  if (batch < 0 || Hq <= 0 || Hkv <= 0) return TA_ERR_INVALID_ARG;
  if (batch > 0 && !seqlens) return TA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return TA_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b)
    if (seqlens[b] < 0) return TA_ERR_INVALID_ARG;
  if (dt != TA_BF16 && dt != TA_F32) return TA_ERR_INVALID_ARG;
  if (!pick_kernel(dt, D, Hq / Hkv, false, ki)) return TA_ERR_UNSUPPORTED;
  return TA_OK;
}

// k and v may be NULL when no token is read (every length 0); nothing dereferences them then.
ta_status check_ptrs(const void* q, const void* k, const void* v, const float* out, const float* lse,
                     bool kv_read) {
  if (!q || !out || !lse) return TA_ERR_INVALID_ARG;
  if (kv_read && (!k || !v)) return TA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return TA_ERR_INVALID_ARG;
  if (!aligned(out, 4) || !aligned(lse, 4)) return TA_ERR_INVALID_ARG;
  return TA_OK;
}

bool any_tokens(const int64_t* seqlens, int batch) {
  for (int b = 0; b < batch; ++b)
    if (seqlens[b] > 0) return true;
  return false;
}

// ------------------------------------------------------------------------------------------
// Launch of a planned decode (workspace body at `body`, error word at `err`)
// ------------------------------------------------------------------------------------------

// A paged cache: pages [num_pages][Hkv][page_size][D], block table rows of `stride` entries.
struct PagedCache {
  const int32_t* table = nullptr;
  int64_t stride = 0;
  int64_t num_pages = 0;
  int log2_page = 0;
};

// n_queries / q_first: query tokens per sequence and the first one this launch covers (the
// kernel instance's G rows per unit are G / (Hq / Hkv) consecutive query tokens).
// Prefix statistics folded into a suffix pass's final write (shared-prefix decode).
struct PrefixFold {
  const float* part = nullptr;  // [chunks][Hkv][rows][stride]
  int chunks = 0, rows = 0, stride = 0;
};

ta_status launch_plan(const Plan& plan, const KernelInfo& ki, const void* q, const void* k, const void* v,
                      float* out, float* lse, int Hq, int Hkv, int D, float scale, ta_dtype dt,
                      const ta_options* opts, uint8_t* body, int* err, cudaStream_t st, int n_queries = 1,
                      int q_first = 0, const PagedCache* pc = nullptr, const PrefixFold* pf = nullptr) {
  const size_t qe = (dt == TA_BF16) ? 2 : 4;
  int log2_heads = 0;
  while ((1 << (log2_heads + 1)) <= Hq / Hkv) ++log2_heads;
  const double s2 = static_cast<double>(scale) * 1.4426950408889634073599246810019;
  ProfileSpan prof(st);
  for (const Group& g : plan.groups) {
    SplitParams p;
    std::memset(&p, 0, sizeof(p));
    const size_t rows0 = static_cast<size_t>(g.b0) * n_queries * Hq;  // first output row of the group
    p.q = static_cast<const uint8_t*>(q) + rows0 * D * qe;
    p.k = k;
    p.v = v;
    p.out = out + rows0 * D;
    p.lse = lse + rows0;
    p.tickets = reinterpret_cast<int*>(body + g.tickets_off);
    p.part = reinterpret_cast<float*>(body + g.part_off);
    p.err = err;
    p.n_tiles_total = g.NT;
    p.wait_limit_ns = 1000LL * ((opts && opts->wait_limit_us > 0) ? opts->wait_limit_us : kDefaultWaitUs);
    p.grid = g.P;
    p.batch = g.nb;
    p.n_kv_heads = Hkv;
    p.n_q_heads = Hq;
    p.scale_log2 = static_cast<float>(s2);
    p.debug_skip_tile = opts ? opts->debug_skip_tile : -1;
    p.unit_aligned = g.unit_aligned ? 1 : 0;
    p.n_queries = n_queries;
    p.q_first = q_first;
    p.log2_heads = log2_heads;
    if (pf) {
      p.pre_part = pf->part + static_cast<int64_t>(g.b0) * (Hq / Hkv) * pf->stride;
      p.pre_chunks = pf->chunks;
      p.pre_rows = pf->rows;
      p.pre_stride = pf->stride;
    }
    if (pc) {
      p.block_table = pc->table + static_cast<int64_t>(g.b0) * pc->stride;
      p.bt_stride = pc->stride;
      p.num_pages = pc->num_pages;
      p.log2_page = pc->log2_page;
    }
    for (int i = 0; i < g.nb; ++i) {
      p.kv_off[i] = g.kv_off[i];
      p.seq_len[i] = g.len[i];
      p.tile_off[i] = g.tile_off[i];
      p.n_tiles[i] = g.n_tiles[i];
    }
    p.tile_off[g.nb] = g.tile_off[g.nb];
    prof.begin();
    ki.fn<<<g.P, ki.threads, ki.smem, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  prof.end();
  return TA_OK;
}

struct DecodeArgs {
  ta_dtype dt;
  const void *q, *k, *v;
  const int64_t* seqlens;
  const int64_t* kv_offsets;
  int batch, Hq, Hkv, D;
  float scale;
  float *out, *lse;
};

// Checks that need no device: options, shape, scale and (when asked) pointers.
ta_status validate(const DecodeArgs& a, const ta_options* opts, bool check_pointers, KernelInfo* ki) {
  ta_status s = check_opts(opts);
  if (s != TA_OK) return s;
  s = check_shape(a.seqlens, a.batch, a.Hq, a.Hkv, a.D, a.dt, ki);
  if (s != TA_OK) return s;
  if (!std::isfinite(a.scale)) return TA_ERR_INVALID_ARG;
  pick_kernel(a.dt, a.D, a.Hq / a.Hkv, use_short_tiles(a.seqlens, a.batch, opts), ki);
  if (check_pointers && a.batch > 0)
    return check_ptrs(a.q, a.k, a.v, a.out, a.lse, any_tokens(a.seqlens, a.batch));
  return TA_OK;
}

// The work plan on the current device (queries SM count and occupancy once).
ta_status plan_for(const DecodeArgs& a, const ta_options* opts, const KernelInfo& ki, Plan* plan) {
  int dev = 0, slots = 1;
  if (a.batch > 0) {
    const ta_status s = resident_ctas(ki, &dev, &slots);
    if (s != TA_OK) return s;
  }
  return build_plan(a.seqlens, a.kv_offsets, a.batch, a.Hkv, a.Hq / a.Hkv, a.D, ki.tile, slots, opts, plan);
}

// Plain bf16 decode with G = 8 query heads per KV head (head_dim 128) runs as the several-query
// form with one query token: its G rows per (sequence, KV head) go to the tensor cores, which
// read each K/V tile once for all of them (the split kernel's G = 8 instances are FP32-issue
// bound).  ta_options.prefix_path 2 keeps the split kernel; 1 sends any bf16 head_dim-128 decode
// to the tensor cores.
bool decode_on_tensor_cores(const DecodeArgs& a, const ta_options* opts) {
  if (a.dt != TA_BF16 || a.D != kBifD || a.kv_offsets != nullptr) return false;
  const int path = opts ? opts->prefix_path : 0;
  return path == 1 || (path == 0 && a.Hq / a.Hkv == 8);
}

ta_status decode_workspace_bytes(const DecodeArgs& a, const ta_options* opts, const KernelInfo& ki, size_t* bytes);

// Decode through the several-query form (defined with it, below); with bytes_only it only
// reports the workspace size.
ta_status decode_tc(const DecodeArgs& a, const ta_options* opts, void* ws, size_t ws_bytes, cudaStream_t st,
                    size_t* bytes_only);

ta_status decode_with_workspace(const DecodeArgs& a, const ta_options* opts, void* ws, size_t ws_bytes,
                                cudaStream_t st) {
  KernelInfo ki;
  Plan plan;
  ta_status s = validate(a, opts, true, &ki);
  if (s != TA_OK) return s;
  if (a.batch == 0) return TA_OK;
  if (decode_on_tensor_cores(a, opts)) return decode_tc(a, opts, ws, ws_bytes, st, nullptr);
  if (!ws || !aligned(ws, kAlign)) return TA_ERR_WORKSPACE;
  s = plan_for(a, opts, ki, &plan);
  if (s != TA_OK) return s;
  if (ws_bytes < kHeaderBytes + plan.body_bytes) return TA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  return launch_plan(plan, ki, a.q, a.k, a.v, a.out, a.lse, a.Hq, a.Hkv, a.D, a.scale, a.dt, opts,
                     base + kHeaderBytes, reinterpret_cast<int*>(base), st);
}

// Allocating form: stream-ordered allocation, zero fill, run, stream-ordered free.
ta_status with_temp_workspace(size_t bytes, cudaStream_t st, ta_status (*run)(void*, size_t, void*, cudaStream_t),
                              void* ctx) {
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, bytes, st);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemsetAsync(ws, 0, bytes, st);
  if (e != cudaSuccess) {
    cudaFreeAsync(ws, st);
    return cuda_fail(e);
  }
  const ta_status s = run(ws, bytes, ctx, st);
  e = cudaFreeAsync(ws, st);
  if (s != TA_OK) return s;
  if (e != cudaSuccess) return cuda_fail(e);
  return TA_OK;
}

// ------------------------------------------------------------------------------------------
// Several query tokens per sequence: passes of G * n' rows per unit (n' query tokens, a power
// of two with G * n' <= 8), each over the whole cache, sharing one workspace in turn.
// ------------------------------------------------------------------------------------------

struct MultiPass {
  int q_first = 0, n_q = 0;
  KernelInfo ki;
  Plan plan;
};

// Either split-KV passes, or the tensor-core form: per launch group of at most kBifMaxSeq
// sequences one bif_prefix_kernel launch in mode 1 (grid chunks x Hkv x sequences) and one
// merge of each unit's 2 * chunks partials.
struct MultiPlan {
  bool tc = false;
  std::vector<MultiPass> passes;
  std::vector<int> chunks;  // tensor-core form: chunks per unit of each launch group
  int rows = 0;
  size_t body = 0;  // workspace bytes after the header
};

ta_status bif_tc_setup(int* sms);
ta_status encode_cache_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows);

ta_status multi_validate(const DecodeArgs& a, int n_queries, const ta_options* opts, bool check_pointers,
                         KernelInfo* ki) {
  if (n_queries < 1) return TA_ERR_INVALID_ARG;
  const ta_status s = validate(a, opts, check_pointers, ki);
  if (s != TA_OK) return s;
  for (int b = 0; b < a.batch; ++b)
    if (a.seqlens[b] < n_queries) return TA_ERR_INVALID_ARG;  // the query tokens are in the cache
  return TA_OK;
}

ta_status multi_plan(const DecodeArgs& a, int n_queries, const ta_options* opts, MultiPlan* mp_out,
                     const PagedCache* pc = nullptr) {
  const int G = a.Hq / a.Hkv;
  MultiPlan& P = *mp_out;
  P = MultiPlan();
  // Tensor-core form: bf16, head_dim 128, 8..128 rows per unit, cache rows addressable by the
  // tensor map's 32-bit coordinates.
  int64_t cache_rows = 0;
  for (int b = 0; b < a.batch; ++b) cache_rows += a.seqlens[b] * a.Hkv;
  if (pc) cache_rows = (pc->num_pages * a.Hkv) << pc->log2_page;
  const int rows = G * n_queries;
  const bool tc_ok = a.dt == TA_BF16 && a.D == kBifD && rows <= kBifRows && cache_rows < (int64_t(1) << 31) &&
                     a.kv_offsets == nullptr;
  const int path = opts ? opts->prefix_path : 0;
  if (path == 1 && !tc_ok) return TA_ERR_UNSUPPORTED;
  if (path == 1 || (path == 0 && tc_ok && rows >= 8)) {
    P.tc = true;
    P.rows = rows;
    int sms = 1;
    if (a.batch > 0) {
      const ta_status s = bif_tc_setup(&sms);
      if (s != TA_OK) return s;
    }
    size_t part = 0;
    for (int b0 = 0; b0 < a.batch; b0 += kBifMaxSeq) {
      const int nb = std::min(kBifMaxSeq, a.batch - b0);
      int64_t max_tiles = 1;
      for (int i = 0; i < nb; ++i) max_tiles = std::max<int64_t>(max_tiles, (a.seqlens[b0 + i] + kBifKeys - 1) / kBifKeys);
      const int64_t c = std::max<int64_t>(1, std::min<int64_t>(sms / (static_cast<int64_t>(nb) * a.Hkv), max_tiles));
      P.chunks.push_back(static_cast<int>(c));
      part = std::max(part, sizeof(float) * static_cast<size_t>(nb) * a.Hkv * c * kBifMT * rows * kBifPartRow);
    }
    P.body = part;
    return TA_OK;
  }
  const bool short_tiles = use_short_tiles(a.seqlens, a.batch, opts);
  for (int j0 = 0; j0 < n_queries;) {
    int nq = 1;
    while (2 * nq <= n_queries - j0 && G * 2 * nq <= 8) nq *= 2;
    MultiPass mp;
    mp.q_first = j0;
    mp.n_q = nq;
    if (!pick_kernel(a.dt, a.D, G * nq, short_tiles, &mp.ki, pc != nullptr)) return TA_ERR_UNSUPPORTED;
    if (pc && mp.ki.tile / (1 << pc->log2_page) + 1 > 32) return TA_ERR_UNSUPPORTED;
    int dev = 0, slots = 1;
    if (a.batch > 0) {
      const ta_status s = resident_ctas(mp.ki, &dev, &slots);
      if (s != TA_OK) return s;
    }
    const ta_status s = build_plan(a.seqlens, a.kv_offsets, a.batch, a.Hkv, G * nq, a.D, mp.ki.tile, slots, opts,
                                   &mp.plan);
    if (s != TA_OK) return s;
    P.body = std::max(P.body, mp.plan.body_bytes);
    P.passes.push_back(mp);
    j0 += nq;
  }
  return TA_OK;
}

ta_status multi_run(const DecodeArgs& a, int n_queries, const ta_options* opts, const MultiPlan& P, void* ws,
                    size_t ws_bytes, cudaStream_t st, const PagedCache* pc = nullptr) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < kHeaderBytes + P.body) return TA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(base);
  if (!P.tc) {
    for (const MultiPass& mp : P.passes) {
      const ta_status s = launch_plan(mp.plan, mp.ki, a.q, a.k, a.v, a.out, a.lse, a.Hq, a.Hkv, a.D, a.scale, a.dt,
                                      opts, base + kHeaderBytes, err, st, n_queries, mp.q_first, pc);
      if (s != TA_OK) return s;
    }
    return TA_OK;
  }
  int64_t cache_rows = 0;
  for (int b = 0; b < a.batch; ++b) cache_rows += a.seqlens[b] * a.Hkv;
  int box_rows = kBifKeys;
  if (pc) {  // the maps cover the page pools; one box per page segment of a key tile
    cache_rows = (pc->num_pages * a.Hkv) << pc->log2_page;
    box_rows = std::min(1 << pc->log2_page, kBifKeys);
  }
  CUtensorMap kmap, vmap;
  ta_status s = encode_cache_map(&kmap, a.k, cache_rows, box_rows);
  if (s != TA_OK) return s;
  s = encode_cache_map(&vmap, a.v, cache_rows, box_rows);
  if (s != TA_OK) return s;
  float* part = reinterpret_cast<float*>(base + kHeaderBytes);
  int64_t row0 = 0;  // tensor-map row of the group's first sequence
  ProfileSpan prof(st);
  for (int b0 = 0; b0 < a.batch; b0 += kBifMaxSeq) {
    const int nb = std::min(kBifMaxSeq, a.batch - b0);
    BifParams bp;
    std::memset(&bp, 0, sizeof(bp));
    const size_t qrow0 = static_cast<size_t>(b0) * n_queries * a.Hq;
    bp.q = static_cast<const uint8_t*>(a.q) + qrow0 * a.D * 2;
    bp.part = part;
    bp.err = err;
    bp.n_samples = nb;
    bp.n_q_heads = a.Hq;
    bp.n_kv_heads = a.Hkv;
    bp.rows_per_head = P.rows;
    for (int i = 0; i < nb; ++i) {
      bp.kv_row0[i] = row0;
      bp.kv_len[i] = a.seqlens[b0 + i];
      row0 += a.seqlens[b0 + i] * a.Hkv;
    }
    bp.n_chunks = P.chunks[b0 / kBifMaxSeq];
    bp.prefix_len = 0;
    bp.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634073599246810019);
    bp.wait_limit_ns = 1000LL * ((opts && opts->wait_limit_us > 0) ? opts->wait_limit_us : kDefaultWaitUs);
    bp.mode = 1;
    bp.n_queries = n_queries;
    bp.debug_skip_tile1 = (opts && opts->debug_skip_tile >= 0 && b0 == 0) ? opts->debug_skip_tile + 1 : 0;
    if (pc) {
      bp.block_table = pc->table + static_cast<int64_t>(b0) * pc->stride;
      bp.bt_stride = pc->stride;
      bp.num_pages = pc->num_pages;
      bp.log2_page = pc->log2_page;
    }
    prof.begin();
    cudaError_t e = launch_bif_prefix(dim3(bp.n_chunks, a.Hkv, nb), kmap, vmap, bp, st);
    if (e != cudaSuccess) return cuda_fail(e);
    if (b0 + kBifMaxSeq >= a.batch) prof.end();
    e = launch_merge_chunks(part, bp.n_chunks, a.Hkv, P.rows, n_queries, a.out + qrow0 * a.D, a.lse + qrow0, nb,
                            a.Hq, err, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return TA_OK;
}

// Workspace of a decode call: the split plan's, or, when the call goes to the tensor cores, the
// larger of that and the tensor-core plan's (a paged call whose page pool is too large for the
// tensor maps falls back to the split plan, so either must fit).
ta_status decode_workspace_bytes(const DecodeArgs& a, const ta_options* opts, const KernelInfo& ki, size_t* bytes) {
  Plan plan;
  ta_status s = plan_for(a, opts, ki, &plan);
  if (s != TA_OK) return s;
  size_t n = kHeaderBytes + plan.body_bytes;
  if (a.batch > 0 && decode_on_tensor_cores(a, opts)) {
    size_t tc = 0;
    s = decode_tc(a, opts, nullptr, 0, nullptr, &tc);
    if (s != TA_OK) return s;
    n = std::max(n, tc);
  }
  *bytes = n;
  return TA_OK;
}

ta_status decode_tc(const DecodeArgs& a, const ta_options* opts, void* ws, size_t ws_bytes, cudaStream_t st,
                    size_t* bytes_only) {
  MultiPlan plan;
  const ta_status s = multi_plan(a, 1, opts, &plan);
  if (s != TA_OK) return s;
  if (bytes_only) {
    *bytes_only = kHeaderBytes + plan.body;
    return TA_OK;
  }
  return multi_run(a, 1, opts, plan, ws, ws_bytes, st);
}

// ------------------------------------------------------------------------------------------
// Bifurcated decode: prefix pass (all samples read the one shared prefix), suffix pass,
// then an exact merge of the two softmax statistics per (sample, query head).
// ------------------------------------------------------------------------------------------

// out = (w_a out_a + w_b out_b) / (w_a + w_b), w_x = e^(lse_x - M), lse = M + ln(w_a + w_b).
__global__ void merge_two_kernel(const float* __restrict__ out_a, const float* __restrict__ lse_a,
                                 const float* __restrict__ out_b, const float* __restrict__ lse_b,
                                 float* __restrict__ out, float* __restrict__ lse, int64_t rows, int D) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * D) return;
  const int64_t r = i / D;
  const int d = static_cast<int>(i % D);
  const float la = lse_a[r], lb = lse_b[r];
  const float M = fmaxf(la, lb);
  float o, l;
  if (M == -INFINITY) {
    o = 0.f;
    l = -INFINITY;
  } else {
    const float wa = (la == -INFINITY) ? 0.f : expf(la - M);
    const float wb = (lb == -INFINITY) ? 0.f : expf(lb - M);
    const float w = wa + wb;
    o = (wa * out_a[i] + wb * out_b[i]) / w;
    l = M + logf(w);
  }
  if (std::isnan(la) || std::isnan(lb)) o = l = __int_as_float(0x7fc00000);
  out[i] = o;
  if (d == 0) lse[r] = l;
}

// Sequence-sharded results: out = sum_s w_s out_s / sum_s w_s, w_s = e^(lse_s - M),
// lse = M + ln sum_s w_s, both sums over the shards in a fixed pairwise tree (a binary
// counter over the shard index).  One thread per output element.
__global__ void merge_shards_kernel(const float* __restrict__ outs, const float* __restrict__ lses, int n_shards,
                                    int64_t rows, int D, float* __restrict__ out, float* __restrict__ lse) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= rows * D) return;
  const int64_t r = i / D;
  const int d = static_cast<int>(i % D);
  float M = -INFINITY;
  bool nan = false;
  for (int sh = 0; sh < n_shards; ++sh) {
    const float l = lses[sh * rows + r];
    nan |= (l != l);
    M = fmaxf(M, l);
  }
  PairwiseSum so, sw;
  for (int sh = 0; sh < n_shards; ++sh) {
    const float l = lses[sh * rows + r];
    const float w = (l == -INFINITY) ? 0.f : expf(l - M);
    sw.push(w);
    so.push(w * outs[(sh * rows + r) * D + d]);
  }
  const float W = sw.result();
  float o = 0.f, lv = -INFINITY;
  if (W > 0.f) {
    o = so.result() / W;
    lv = M + logf(W);
  }
  if (nan) o = lv = __int_as_float(0x7fc00000);
  out[i] = o;
  if (d == 0) lse[r] = lv;
}

struct BifArgs {
  const void *q, *kp, *vp, *ks, *vs;
  int64_t P;
  const int64_t* suffix_lens;
  int N, Hq, Hkv, D;
  float scale;
  float *out, *lse;
};

struct BifPlan {
  KernelInfo ki, ki_suffix;  // split kernel of the prefix pass (per sample) and of the suffix pass
  Plan prefix, suffix;
  std::vector<int64_t> prefix_lens, prefix_offs;
  size_t scratch_off = 0, body_off = 0, suffix_off = 0, total = 0;
  // tensor-core prefix pass
  bool tc = false;
  int mtiles = 0, chunks = 0, rows_per_head = 0;
  size_t part_off = 0;
  bool short_suffix = false;  // suffix pass on the short-unit kernel (tensor-core prefix pass only)
  int sms = 0;
};

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows][128] bf16 matrix, boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool encode_kv_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows = kBifKeys) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn || rows <= 0 || rows >= (int64_t(1) << 31)) return false;  // tile rows are 32-bit coordinates
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kBifD), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kBifD) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The whole packed cache as one [rows][128] bf16 matrix for the tensor-core passes.
ta_status encode_cache_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows) {
  if (rows <= 0) rows = 1;  // no key is read; the map only has to be valid
  return encode_kv_map(map, base, rows, box_rows) ? TA_OK : TA_ERR_UNSUPPORTED;
}

ta_status bif_tc_setup(int* sms) {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::call_once(once, [] {
    err = bif_prefix_set_smem_limit();
  });
  if (err != cudaSuccess) return cuda_fail(err);
  return TA_OK;
}

ta_status bif_validate(const BifArgs& a, const ta_options* opts, bool check_pointers, KernelInfo* ki) {
  if (a.P < 0 || a.N < 0) return TA_ERR_INVALID_ARG;
  if (a.N > 0 && !a.suffix_lens) return TA_ERR_INVALID_ARG;
  const int64_t plen = a.P;
  DecodeArgs probe{TA_BF16, a.q, a.kp, a.vp, &plen, nullptr, a.N > 0 ? 1 : 0, a.Hq, a.Hkv, a.D, a.scale,
                   a.out, a.lse};
  ta_status s = validate(probe, opts, check_pointers, ki);
  if (s != TA_OK) return s;
  for (int n = 0; n < a.N; ++n)
    if (a.suffix_lens[n] < 0) return TA_ERR_INVALID_ARG;
  if (check_pointers && a.N > 0) {
    if (any_tokens(a.suffix_lens, a.N) && (!a.ks || !a.vs)) return TA_ERR_INVALID_ARG;
    if (!aligned(a.ks, 16) || !aligned(a.vs, 16)) return TA_ERR_INVALID_ARG;
  }
  return TA_OK;
}

ta_status bif_plan(const BifArgs& a, const ta_options* opts, const KernelInfo& ki, BifPlan* bp) {
  bp->prefix_lens.assign(a.N, a.P);
  bp->prefix_offs.assign(a.N, 0);
  bp->ki = ki;
  bp->ki_suffix = ki;
  if (a.N > 0) {
    pick_kernel(TA_BF16, a.D, a.Hq / a.Hkv, use_short_tiles(bp->prefix_lens.data(), a.N, opts), &bp->ki);
    pick_kernel(TA_BF16, a.D, a.Hq / a.Hkv, use_short_tiles(a.suffix_lens, a.N, opts), &bp->ki_suffix);
  }
  DecodeArgs pre{TA_BF16, a.q, a.kp, a.vp, bp->prefix_lens.data(), bp->prefix_offs.data(), a.N, a.Hq, a.Hkv, a.D,
                 a.scale, a.out, a.lse};
  ta_status s = plan_for(pre, opts, bp->ki, &bp->prefix);
  if (s != TA_OK) return s;
  DecodeArgs suf{TA_BF16, a.q, a.ks, a.vs, a.suffix_lens, nullptr, a.N, a.Hq, a.Hkv, a.D, a.scale, a.out, a.lse};
  s = plan_for(suf, opts, bp->ki_suffix, &bp->suffix);
  if (s != TA_OK) return s;
  const size_t rows = static_cast<size_t>(a.N) * a.Hq;
  bp->scratch_off = kHeaderBytes;
  bp->body_off = align_up(bp->scratch_off + 2 * sizeof(float) * rows * (a.D + 1), kAlign);
  // Each pass keeps its own tickets and partials: one pass's partials must never sit
  // where the other pass expects zeroed tickets.
  bp->suffix_off = align_up(bp->body_off + bp->prefix.body_bytes, kAlign);
  bp->total = bp->suffix_off + bp->suffix.body_bytes;
  // Tensor-core prefix pass: one CTA per (128-row tile, prefix chunk, KV head).
  const int path = opts ? opts->prefix_path : 0;
  const bool tc_shape = a.D == kBifD && a.P > 0;
  if (path == 1 && !tc_shape) return TA_ERR_UNSUPPORTED;
  if (path != 2 && tc_shape && a.N > 0) {
    int sms = 0;
    s = bif_tc_setup(&sms);
    if (s != TA_OK) return s;
    bp->tc = true;
    bp->sms = sms;
    bp->rows_per_head = a.N * (a.Hq / a.Hkv);
    bp->mtiles = (bp->rows_per_head + kBifMT * kBifRows - 1) / (kBifMT * kBifRows);  // CTAs per (chunk, head)
    const int64_t tiles = (a.P + kBifKeys - 1) / kBifKeys;
    int64_t chunks = sms / (static_cast<int64_t>(bp->mtiles) * a.Hkv);
    chunks = std::max<int64_t>(1, std::min<int64_t>(chunks, tiles));
    bp->chunks = static_cast<int>(chunks);
    bp->part_off = align_up(bp->total, kAlign);
    bp->total = bp->part_off +
                sizeof(float) * static_cast<size_t>(chunks) * a.Hkv * bp->rows_per_head * kBifPartRow;
    // Many short suffixes: one CTA per (sample, KV head) keeps every unit resident at once.
    int64_t longest = 0;
    for (int n = 0; n < a.N; ++n) longest = std::max(longest, a.suffix_lens[n]);
    const int tiles_opt = opts ? opts->split_tiles : 0;
    bp->short_suffix = a.D == 128 && chunks <= kShortMaxChunks &&
                       (tiles_opt == 3 ||
                        (tiles_opt == 0 && static_cast<int64_t>(a.N) * a.Hkv >= sms && longest <= kShortMaxLen));
  }
  return TA_OK;
}

// The suffix pass on the short-unit kernel: one launch per 128 samples, the first of them
// allowed to start while the prefix pass (the stream's previous kernel) still runs.
ta_status launch_short(const BifArgs& a, const ta_options* opts, int sms, const PrefixFold& pf, int* err,
                       cudaStream_t st) {
  const int G = a.Hq / a.Hkv;
  int64_t off = 0;
  for (int b0 = 0; b0 < a.N; b0 += kShortMaxSeq) {
    const int nb = std::min(kShortMaxSeq, a.N - b0);
    ShortParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.q = static_cast<const __nv_bfloat16*>(a.q) + static_cast<int64_t>(b0) * a.Hq * a.D;
    sp.k = static_cast<const __nv_bfloat16*>(a.ks);
    sp.v = static_cast<const __nv_bfloat16*>(a.vs);
    sp.out = a.out + static_cast<int64_t>(b0) * a.Hq * a.D;
    sp.lse = a.lse + static_cast<int64_t>(b0) * a.Hq;
    sp.err = err;
    sp.pre_part = pf.part + static_cast<int64_t>(b0) * G * pf.stride;
    sp.pre_chunks = pf.chunks;
    sp.pre_rows = pf.rows;
    sp.pre_stride = pf.stride;
    sp.n_kv_heads = a.Hkv;
    sp.n_q_heads = a.Hq;
    sp.n_seq = nb;
    sp.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634073599246810019);
    sp.wait_limit_ns = 1000LL * ((opts && opts->wait_limit_us > 0) ? opts->wait_limit_us : kDefaultWaitUs);
    sp.debug_skip_stage1 = (opts && b0 == 0) ? opts->debug_skip_stage : 0;
    for (int i = 0; i < nb; ++i) {
      sp.kv_off[i] = off;
      sp.seq_len[i] = a.suffix_lens[b0 + i];
      off += a.suffix_lens[b0 + i] * a.Hkv * a.D;
    }
    const cudaError_t e = launch_short_decode(G, sp, sms, opts ? opts->num_ctas : 0, b0 == 0, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return TA_OK;
}

ta_status bif_run(const BifArgs& a, const ta_options* opts, const BifPlan& bp, void* ws, size_t ws_bytes,
                  cudaStream_t st) {
  if (a.N == 0) return TA_OK;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < bp.total) return TA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(base);
  const size_t rows = static_cast<size_t>(a.N) * a.Hq;
  float* out_p = reinterpret_cast<float*>(base + bp.scratch_off);
  float* out_s = out_p + rows * a.D;
  float* lse_p = out_s + rows * a.D;
  float* lse_s = lse_p + rows;
  ta_status s;
  if (bp.tc) {
    CUtensorMap kmap, vmap;
    const int64_t kv_rows = static_cast<int64_t>(a.Hkv) * a.P;
    const bool maps = encode_kv_map(&kmap, a.kp, kv_rows) && encode_kv_map(&vmap, a.vp, kv_rows);
    if (maps) {
      BifParams bpp;
      std::memset(&bpp, 0, sizeof(bpp));  // mode 0, contiguous prefix: no block table
      bpp.q = a.q;
      bpp.part = reinterpret_cast<float*>(base + bp.part_off);
      bpp.err = err;
      bpp.n_samples = a.N;
      bpp.n_q_heads = a.Hq;
      bpp.n_kv_heads = a.Hkv;
      bpp.rows_per_head = bp.rows_per_head;
      bpp.n_chunks = bp.chunks;
      bpp.prefix_len = a.P;
      bpp.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634073599246810019);
      bpp.wait_limit_ns = 1000LL * ((opts && opts->wait_limit_us > 0) ? opts->wait_limit_us : kDefaultWaitUs);
      bpp.debug_skip_tile1 = (opts && opts->debug_skip_tile >= 0) ? opts->debug_skip_tile + 1 : 0;
      const dim3 grid(bp.mtiles, bp.chunks, a.Hkv);
      ProfileSpan prof(st);
      prof.begin();
      cudaError_t e = launch_bif_prefix(grid, kmap, vmap, bpp, st);
      if (e != cudaSuccess) return cuda_fail(e);
      prof.end();
      const cudaEvent_t saved_start = g_prof_start, saved_stop = g_prof_stop;
      g_prof_start = g_prof_stop = nullptr;  // the suffix pass is not the main kernel here
      // The suffix pass folds the prefix chunks' statistics into each row as it writes it.
      PrefixFold pf;
      pf.part = bpp.part;
      pf.chunks = bp.chunks;
      pf.rows = bp.rows_per_head;
      pf.stride = kBifPartRow;
      if (bp.short_suffix)
        s = launch_short(a, opts, bp.sms, pf, err, st);
      else
        s = launch_plan(bp.suffix, bp.ki_suffix, a.q, a.ks, a.vs, a.out, a.lse, a.Hq, a.Hkv, a.D, a.scale, TA_BF16,
                        opts, base + bp.suffix_off, err, st, 1, 0, nullptr, &pf);
      g_prof_start = saved_start;
      g_prof_stop = saved_stop;
      return s;
    }
    if (opts && opts->prefix_path == 1) return TA_ERR_UNSUPPORTED;
  }
  s = launch_plan(bp.prefix, bp.ki, a.q, a.kp, a.vp, out_p, lse_p, a.Hq, a.Hkv, a.D, a.scale, TA_BF16, opts,
                  base + bp.body_off, err, st);
  if (s != TA_OK) return s;
  s = launch_plan(bp.suffix, bp.ki_suffix, a.q, a.ks, a.vs, out_s, lse_s, a.Hq, a.Hkv, a.D, a.scale, TA_BF16, opts,
                  base + bp.suffix_off, err, st);
  if (s != TA_OK) return s;
  const int64_t n = static_cast<int64_t>(rows) * a.D;
  merge_two_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(out_p, lse_p, out_s, lse_s, a.out,
                                                                          a.lse, static_cast<int64_t>(rows), a.D);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return TA_OK;
}

}  // namespace
}  // namespace ta

using namespace ta;

extern "C" {

const char* tree_attn_status_string(ta_status s) {
  switch (s) {
    case TA_OK: return "ok";
    case TA_ERR_INVALID_ARG: return "invalid argument";
    case TA_ERR_UNSUPPORTED: return "unsupported shape";
    case TA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case TA_ERR_CUDA: return "CUDA error";
    case TA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case TA_ERR_SCRATCH_LIMIT: return "needs more scratch than the fixed 4 MiB no-allocation buffer holds";
    case TA_ERR_BAD_PAGE: return "a block-table entry is outside [0, num_pages)";
  }
  return "unknown status";
}

int32_t tree_attn_last_cuda_error(void) { return g_last_cuda_error; }

void tree_attn_profile_events(void* start, void* stop) {
  g_prof_start = static_cast<cudaEvent_t>(start);
  g_prof_stop = static_cast<cudaEvent_t>(stop);
}

ta_status tree_attn_workspace_size(const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                   int32_t head_dim, ta_dtype dtype, const ta_options* opts, size_t* bytes) {
  if (!bytes) return TA_ERR_INVALID_ARG;
  DecodeArgs a{dtype, nullptr, nullptr, nullptr, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               1.0f, nullptr, nullptr};
  KernelInfo ki;
  ta_status s = validate(a, opts, false, &ki);
  if (s != TA_OK) return s;
  return decode_workspace_bytes(a, opts, ki, bytes);
}

ta_status tree_attn_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < kHeaderBytes) return TA_ERR_WORKSPACE;
  const cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TA_OK;
}

ta_status tree_attn_decode_ex(ta_dtype dtype, const void* q, const void* k_cache, const void* v_cache,
                              const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                              int32_t head_dim, float scale, float* out, float* lse, const ta_options* opts,
                              void* workspace, size_t workspace_bytes, void* stream) {
  DecodeArgs a{dtype, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  return decode_with_workspace(a, opts, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

namespace {
struct PlainCtx {
  DecodeArgs a;
};
ta_status plain_run(void* ws, size_t bytes, void* ctx, cudaStream_t st) {
  return decode_with_workspace(static_cast<PlainCtx*>(ctx)->a, nullptr, ws, bytes, st);
}
ta_status decode_alloc(const DecodeArgs& a, cudaStream_t st) {
  KernelInfo ki;
  Plan plan;
  ta_status s = validate(a, nullptr, true, &ki);
  if (s != TA_OK) return s;
  if (a.batch == 0) return TA_OK;
  size_t bytes = 0;
  s = decode_workspace_bytes(a, nullptr, ki, &bytes);
  if (s != TA_OK) return s;
  PlainCtx ctx{a};
  return with_temp_workspace(bytes, st, &plain_run, &ctx);
}
}  // namespace

ta_status tree_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                           int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale,
                           float* out, float* lse, void* stream) {
  DecodeArgs a{TA_BF16, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  return decode_alloc(a, static_cast<cudaStream_t>(stream));
}

ta_status tree_attn_decode_f32(const float* q, const float* k_cache, const float* v_cache, const int64_t* seqlens,
                               int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale,
                               float* out, float* lse, void* stream) {
  DecodeArgs a{TA_F32, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  return decode_alloc(a, static_cast<cudaStream_t>(stream));
}

ta_status tree_attn_bifurcated_workspace_size(int64_t prefix_len, const int64_t* suffix_lens, int32_t n_samples,
                                              int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                              const ta_options* opts, size_t* bytes) {
  if (!bytes) return TA_ERR_INVALID_ARG;
  BifArgs a{nullptr, nullptr, nullptr, nullptr, nullptr, prefix_len, suffix_lens, n_samples, n_q_heads,
            n_kv_heads, head_dim, 1.0f, nullptr, nullptr};
  KernelInfo ki;
  ta_status s = bif_validate(a, opts, false, &ki);
  if (s != TA_OK) return s;
  BifPlan bp;
  s = bif_plan(a, opts, ki, &bp);
  if (s != TA_OK) return s;
  *bytes = bp.total;
  return TA_OK;
}

ta_status tree_attn_decode_bifurcated_ex(const void* q, const void* k_prefix, const void* v_prefix,
                                         int64_t prefix_len, const void* k_suffix, const void* v_suffix,
                                         const int64_t* suffix_lens, int32_t n_samples, int32_t n_q_heads,
                                         int32_t n_kv_heads, int32_t head_dim, float scale, float* out, float* lse,
                                         const ta_options* opts, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  BifArgs a{q, k_prefix, v_prefix, k_suffix, v_suffix, prefix_len, suffix_lens, n_samples, n_q_heads,
            n_kv_heads, head_dim, scale, out, lse};
  KernelInfo ki;
  ta_status s = bif_validate(a, opts, true, &ki);
  if (s != TA_OK || n_samples == 0) return s;
  if (!workspace || !aligned(workspace, kAlign)) return TA_ERR_WORKSPACE;
  BifPlan bp;
  s = bif_plan(a, opts, ki, &bp);
  if (s != TA_OK) return s;
  return bif_run(a, opts, bp, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

namespace {
struct BifCtx {
  BifArgs a;
  const BifPlan* bp;
};
ta_status bif_alloc_run(void* ws, size_t bytes, void* ctx, cudaStream_t st) {
  BifCtx* c = static_cast<BifCtx*>(ctx);
  return bif_run(c->a, nullptr, *c->bp, ws, bytes, st);
}
}  // namespace

ta_status tree_attn_decode_bifurcated(const void* q, const void* k_prefix, const void* v_prefix, int64_t prefix_len,
                                      const void* k_suffix, const void* v_suffix, const int64_t* suffix_lens,
                                      int32_t n_samples, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                      float scale, float* out, float* lse, void* stream) {
  BifArgs a{q, k_prefix, v_prefix, k_suffix, v_suffix, prefix_len, suffix_lens, n_samples, n_q_heads,
            n_kv_heads, head_dim, scale, out, lse};
  KernelInfo ki;
  ta_status s = bif_validate(a, nullptr, true, &ki);
  if (s != TA_OK || n_samples == 0) return s;
  BifPlan bp;
  s = bif_plan(a, nullptr, ki, &bp);
  if (s != TA_OK) return s;
  BifCtx ctx{a, &bp};
  return with_temp_workspace(bp.total, static_cast<cudaStream_t>(stream), &bif_alloc_run, &ctx);
}

ta_status tree_attn_multi_workspace_size(const int64_t* seqlens, int32_t batch, int32_t n_queries,
                                         int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, ta_dtype dtype,
                                         const ta_options* opts, size_t* bytes) {
  if (!bytes) return TA_ERR_INVALID_ARG;
  DecodeArgs a{dtype, nullptr, nullptr, nullptr, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               1.0f, nullptr, nullptr};
  KernelInfo ki;
  ta_status s = multi_validate(a, n_queries, opts, false, &ki);
  if (s != TA_OK) return s;
  MultiPlan plan;
  s = multi_plan(a, n_queries, opts, &plan);
  if (s != TA_OK) return s;
  *bytes = kHeaderBytes + plan.body;
  return TA_OK;
}

ta_status tree_attn_decode_multi_ex(ta_dtype dtype, const void* q, const void* k_cache, const void* v_cache,
                                    const int64_t* seqlens, int32_t batch, int32_t n_queries, int32_t n_q_heads,
                                    int32_t n_kv_heads, int32_t head_dim, float scale, float* out, float* lse,
                                    const ta_options* opts, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  DecodeArgs a{dtype, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  KernelInfo ki;
  ta_status s = multi_validate(a, n_queries, opts, true, &ki);
  if (s != TA_OK || batch == 0) return s;
  MultiPlan plan;
  s = multi_plan(a, n_queries, opts, &plan);
  if (s != TA_OK) return s;
  return multi_run(a, n_queries, opts, plan, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

namespace {
struct MultiCtx {
  DecodeArgs a;
  int n_queries;
  const MultiPlan* plan;
};
ta_status multi_alloc_run(void* ws, size_t bytes, void* ctx, cudaStream_t st) {
  MultiCtx* c = static_cast<MultiCtx*>(ctx);
  return multi_run(c->a, c->n_queries, nullptr, *c->plan, ws, bytes, st);
}
}  // namespace

ta_status tree_attn_decode_multi(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                                 int32_t batch, int32_t n_queries, int32_t n_q_heads, int32_t n_kv_heads,
                                 int32_t head_dim, float scale, float* out, float* lse, void* stream) {
  DecodeArgs a{TA_BF16, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  KernelInfo ki;
  ta_status s = multi_validate(a, n_queries, nullptr, true, &ki);
  if (s != TA_OK || batch == 0) return s;
  MultiPlan plan;
  s = multi_plan(a, n_queries, nullptr, &plan);
  if (s != TA_OK) return s;
  MultiCtx ctx{a, n_queries, &plan};
  return with_temp_workspace(kHeaderBytes + plan.body, static_cast<cudaStream_t>(stream), &multi_alloc_run, &ctx);
}

ta_status tree_attn_decode_multi_paged_ex(ta_dtype dtype, const void* q, const void* k_pages, const void* v_pages,
                                          int64_t num_pages, int32_t page_size, const int32_t* block_table,
                                          int64_t block_table_stride, const int64_t* seqlens, int32_t batch,
                                          int32_t n_queries, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          float scale, float* out, float* lse, const ta_options* opts,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  DecodeArgs a{dtype, q, k_pages, v_pages, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  if (page_size < 16 || page_size > 65536 || (page_size & (page_size - 1)) != 0 || num_pages < 0)
    return TA_ERR_INVALID_ARG;
  PagedCache pc{block_table, block_table_stride, num_pages, 0};
  while ((1 << pc.log2_page) < page_size) ++pc.log2_page;
  KernelInfo ki;
  ta_status s = multi_validate(a, n_queries, opts, true, &ki);
  if (s != TA_OK || batch == 0) return s;
  int64_t max_blocks = 0;
  for (int b = 0; b < batch; ++b) max_blocks = std::max<int64_t>(max_blocks, (seqlens[b] + page_size - 1) / page_size);
  if (block_table_stride < max_blocks || num_pages < 1 || !block_table ||
      (reinterpret_cast<uintptr_t>(block_table) & 3) != 0)
    return TA_ERR_INVALID_ARG;
  MultiPlan plan;
  s = multi_plan(a, n_queries, opts, &plan, &pc);
  if (s != TA_OK) return s;
  return multi_run(a, n_queries, opts, plan, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &pc);
}

namespace {
struct PagedArgs {
  DecodeArgs a;
  PagedCache pc;
};

ta_status paged_validate(const DecodeArgs& a, const PagedCache& pc, int32_t page_size, const ta_options* opts,
                         bool check_pointers, KernelInfo* ki, PagedCache* out) {
  if (page_size < 16 || page_size > 65536 || (page_size & (page_size - 1)) != 0) return TA_ERR_INVALID_ARG;
  if (pc.num_pages < 0) return TA_ERR_INVALID_ARG;
  *out = pc;
  out->log2_page = 0;
  while ((1 << out->log2_page) < page_size) ++out->log2_page;
  ta_status s = validate(a, opts, check_pointers, ki);
  if (s != TA_OK) return s;
  pick_kernel(a.dt, a.D, a.Hq / a.Hkv, use_short_tiles(a.seqlens, a.batch, opts), ki, true);
  int64_t max_blocks = 0;
  for (int b = 0; b < a.batch; ++b) max_blocks = std::max<int64_t>(max_blocks, (a.seqlens[b] + page_size - 1) / page_size);
  if (max_blocks > 0 && (pc.stride < max_blocks || pc.num_pages < 1)) return TA_ERR_INVALID_ARG;
  // A tile touches at most tile / page_size + 1 pages, one producer lane each.
  if (ki->tile / page_size + 1 > 32) return TA_ERR_UNSUPPORTED;
  if (check_pointers && max_blocks > 0 && (!pc.table || (reinterpret_cast<uintptr_t>(pc.table) & 3) != 0))
    return TA_ERR_INVALID_ARG;
  return TA_OK;
}

ta_status paged_run(const PagedArgs& pa, const ta_options* opts, void* ws, size_t ws_bytes, cudaStream_t st) {
  const DecodeArgs& a = pa.a;
  KernelInfo ki;
  PagedCache pc;
  ta_status s = paged_validate(a, pa.pc, 1 << pa.pc.log2_page, opts, true, &ki, &pc);
  if (s != TA_OK) return s;
  if (a.batch == 0) return TA_OK;
  if (!ws || !aligned(ws, kAlign)) return TA_ERR_WORKSPACE;
  if (decode_on_tensor_cores(a, opts)) {  // G = 8 (or forced): the paged tensor-core form, one query token
    if (!pc.table || (reinterpret_cast<uintptr_t>(pc.table) & 3) != 0) return TA_ERR_INVALID_ARG;
    MultiPlan mp;
    s = multi_plan(a, 1, opts, &mp, &pc);
    if (s != TA_OK) return s;
    return multi_run(a, 1, opts, mp, ws, ws_bytes, st, &pc);
  }
  Plan plan;
  s = plan_for(a, opts, ki, &plan);
  if (s != TA_OK) return s;
  if (ws_bytes < kHeaderBytes + plan.body_bytes) return TA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  return launch_plan(plan, ki, a.q, a.k, a.v, a.out, a.lse, a.Hq, a.Hkv, a.D, a.scale, a.dt, opts,
                     base + kHeaderBytes, reinterpret_cast<int*>(base), st, 1, 0, &pc);
}

ta_status paged_alloc_run(void* ws, size_t bytes, void* ctx, cudaStream_t st) {
  return paged_run(*static_cast<PagedArgs*>(ctx), nullptr, ws, bytes, st);
}
}  // namespace

ta_status tree_attn_decode_paged_ex(ta_dtype dtype, const void* q, const void* k_pages, const void* v_pages,
                                    int64_t num_pages, int32_t page_size, const int32_t* block_table,
                                    int64_t block_table_stride, const int64_t* seqlens, int32_t batch,
                                    int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale, float* out,
                                    float* lse, const ta_options* opts, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  PagedArgs pa{DecodeArgs{dtype, q, k_pages, v_pages, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
                          scale, out, lse},
               PagedCache{block_table, block_table_stride, num_pages, 0}};
  if (page_size < 16 || (page_size & (page_size - 1)) != 0) return TA_ERR_INVALID_ARG;
  while ((1 << pa.pc.log2_page) < page_size) ++pa.pc.log2_page;
  return paged_run(pa, opts, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

ta_status tree_attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, int64_t num_pages,
                                 int32_t page_size, const int32_t* block_table, int64_t block_table_stride,
                                 const int64_t* seqlens, int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                 int32_t head_dim, float scale, float* out, float* lse, void* stream) {
  PagedArgs pa{DecodeArgs{TA_BF16, q, k_pages, v_pages, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
                          scale, out, lse},
               PagedCache{block_table, block_table_stride, num_pages, 0}};
  if (page_size < 16 || (page_size & (page_size - 1)) != 0) return TA_ERR_INVALID_ARG;
  while ((1 << pa.pc.log2_page) < page_size) ++pa.pc.log2_page;
  KernelInfo ki;
  PagedCache pc;
  ta_status s = paged_validate(pa.a, pa.pc, page_size, nullptr, true, &ki, &pc);
  if (s != TA_OK || batch == 0) return s;
  size_t bytes = 0;
  s = decode_workspace_bytes(pa.a, nullptr, ki, &bytes);
  if (s != TA_OK) return s;
  return with_temp_workspace(bytes, static_cast<cudaStream_t>(stream), &paged_alloc_run, &pa);
}

// ------------------------------------------------------------------------------------------
// Decode without allocation: the workspace is a fixed array in the library's device memory.
// ------------------------------------------------------------------------------------------

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a stand-in for the symbol, not a device
// address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  Looked up again on every call
// made outside stream capture (so an address from before a device reset is never reused);
// inside a capture the address from the last uncaptured call on this device is used.
ta_status noalloc_scratch_address(cudaStream_t st, void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(mu);
  if (cap == cudaStreamCaptureStatusNone || addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    addr[dev] = p;
  }
  *out = addr[dev];
  return TA_OK;
}

}  // namespace

ta_status tree_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int64_t* seqlens,
                                   int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                   float scale, float* out, float* lse, void* stream) {
  DecodeArgs a{TA_BF16, q, k_cache, v_cache, seqlens, nullptr, batch, n_q_heads, n_kv_heads, head_dim,
               scale, out, lse};
  KernelInfo ki;
  Plan plan;
  ta_status s = validate(a, nullptr, true, &ki);
  if (s != TA_OK) return s;
  if (a.batch == 0) return TA_OK;
  s = plan_for(a, nullptr, ki, &plan);
  if (s != TA_OK) return s;
  const size_t need = kHeaderBytes + plan.body_bytes;
  if (need > kNoAllocScratchBytes) return TA_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = noalloc_scratch_address(st, &ws);
  if (s != TA_OK) return s;
  // The array keeps whatever the previous call left: clear the error word and the tickets.
  uint8_t* base = static_cast<uint8_t*>(ws);
  cudaError_t e = cudaMemsetAsync(base, 0, kHeaderBytes, st);
  for (const Group& g : plan.groups) {
    if (e != cudaSuccess) break;
    e = cudaMemsetAsync(base + kHeaderBytes + g.tickets_off, 0, sizeof(int) * static_cast<size_t>(g.nb) * n_kv_heads,
                        st);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return launch_plan(plan, ki, a.q, a.k, a.v, a.out, a.lse, a.Hq, a.Hkv, a.D, a.scale, a.dt, nullptr,
                     base + kHeaderBytes, reinterpret_cast<int*>(base), st);
}

ta_status tree_attn_merge_shards(const float* outs, const float* lses, int32_t n_shards, int64_t rows,
                                 int32_t head_dim, float* out, float* lse, void* stream) {
  if (n_shards < 1 || n_shards > 65536 || rows < 0 || head_dim <= 0) return TA_ERR_INVALID_ARG;
  if (rows == 0) return TA_OK;
  if (!outs || !lses || !out || !lse) return TA_ERR_INVALID_ARG;
  if (!aligned(outs, 4) || !aligned(lses, 4) || !aligned(out, 4) || !aligned(lse, 4)) return TA_ERR_INVALID_ARG;
  const int64_t n = rows * head_dim;
  merge_shards_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      outs, lses, n_shards, rows, head_dim, out, lse);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return TA_OK;
}

ta_status tree_attn_anchor_prefill(const void* q, const void* k, const void* v, int64_t seq_len, int64_t block_size,
                                   int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, float scale, float* out,
                                   float* lse, const ta_options* opts, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  ta_status s = check_opts(opts);
  if (s != TA_OK) return s;
  if (seq_len < 0 || block_size <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 ||
      !std::isfinite(scale))
    return TA_ERR_INVALID_ARG;
  const int G = n_q_heads / n_kv_heads;
  if (head_dim != kBifD || (G != 1 && G != 2 && G != 4 && G != 8) || block_size % kBifKeys != 0 ||
      static_cast<int64_t>(n_kv_heads) * seq_len >= (int64_t(1) << 31))
    return TA_ERR_UNSUPPORTED;
  if (seq_len == 0) return TA_OK;
  if (!q || !k || !v || !out || !lse) return TA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
    return TA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, kAlign) || workspace_bytes < kHeaderBytes) return TA_ERR_WORKSPACE;
  int sms = 0;
  s = bif_tc_setup(&sms);
  if (s != TA_OK) return s;
  CUtensorMap kmap, vmap;
  const int64_t rows = static_cast<int64_t>(n_kv_heads) * seq_len;
  s = encode_cache_map(&kmap, k, rows, kBifKeys);
  if (s != TA_OK) return s;
  s = encode_cache_map(&vmap, v, rows, kBifKeys);
  if (s != TA_OK) return s;
  BifParams bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.q = q;
  bp.err = static_cast<int*>(workspace);
  bp.n_samples = 1;
  bp.n_q_heads = n_q_heads;
  bp.n_kv_heads = n_kv_heads;
  bp.n_pos = kBifRows / G;
  bp.rows_per_head = kBifRows;
  bp.n_chunks = 1;
  bp.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634073599246810019);
  bp.wait_limit_ns = 1000LL * ((opts && opts->wait_limit_us > 0) ? opts->wait_limit_us : kDefaultWaitUs);
  bp.mode = 2;
  bp.ctx_len = seq_len;
  bp.block_size = block_size;
  bp.out = out;
  bp.lse = lse;
  bp.debug_skip_tile1 = (opts && opts->debug_skip_tile >= 0) ? opts->debug_skip_tile + 1 : 0;
  const int64_t n_tiles = (seq_len + bp.n_pos - 1) / bp.n_pos;
  ProfileSpan prof(static_cast<cudaStream_t>(stream));
  prof.begin();
  const cudaError_t e = launch_bif_prefix(dim3(static_cast<unsigned>(n_tiles), n_kv_heads, 1), kmap, vmap, bp,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  prof.end();
  return TA_OK;
}

ta_status tree_attn_check(const void* ws, void* stream) {
  if (!ws || !aligned(ws, kAlign)) return TA_ERR_WORKSPACE;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int word = 0;
  e = cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (word == 0) return TA_OK;
  return word == kErrBadPage ? TA_ERR_BAD_PAGE : TA_ERR_TIMEOUT;
}

ta_status tree_attn_noalloc_check(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  void* ws = nullptr;
  const ta_status s = noalloc_scratch_address(st, &ws);
  if (s != TA_OK) return s;
  return tree_attn_check(ws, stream);
}

}  // extern "C"
