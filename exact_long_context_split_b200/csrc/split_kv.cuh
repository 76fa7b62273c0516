// Split-KV decode attention: one persistent CTA per SM streams an equal share of
// the whole job's KV tiles through a 4-stage shared-memory ring (bulk copies on
// the TMA engine), computes exp2-domain online-softmax statistics (m, l, o) for
// the G query heads that share each KV head, and merges the statistics of the
// CTAs that shared a (sequence, KV head) in a fixed pairwise tree.
//
// Method: "Attention acceleration" concept page (compassingai.com), Technical
// principles part 1 (S = QK^T/sqrt(d_k), P = softmax(S), O = PV) and part 2.1
// (online softmax: m_new = max(m_old, m_block), l_new = l_old e^{m_old-m_new} +
// sum e^{x-m_new}, O rescaled alike; kept unnormalised here); Tree Attention
// article (m.srwj168.com.cn), "The energy view of attention" (max and
// logsumexp are associative, so partial results combine in any tree).
//
// Work split (one launch): the (sequence, KV head) units are laid end to end as
// a line of NT tiles of TILE tokens; CTA i takes tiles [i*NT/P, (i+1)*NT/P).  A
// CTA that crosses a unit boundary emits one partial per unit it touched.  CTA i
// writes unit u's partial to slot i + u: along the line both i and u only grow,
// so i + u is unique, and unit u's partials sit in consecutive slots.
#pragma once
#include <cuda_bf16.h>

#include <cmath>
#include <cstdint>

#include "ptx.cuh"

namespace ta {

constexpr int kMaxSeqPerLaunch = 128;
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLn2 = 0.693147180559945309f;
// Lazy rescaling: a new score replaces the running max only when it exceeds it
// by more than this (log2 units), so p = 2^(x - m) <= 2^8; the final division
// by l cancels whichever reference max was used.
constexpr float kRescaleThreshold = 8.0f;

// Error codes recorded in the workspace error word.
constexpr int kErrConsumerWait = 1;
constexpr int kErrProducerWait = 2;
constexpr int kErrDrainWait = 3;
constexpr int kErrBadPage = 8;  // a block-table entry outside [0, num_pages): nothing was read for it

struct SplitParams {
  const void* q;   // [B][Hq][D], this launch's first sequence
  const void* k;   // cache base; kv_off[b] is relative to it
  const void* v;
  float* out;      // [B][Hq][D]
  float* lse;      // [B][Hq]
  int* tickets;    // [B * Hkv], zero between calls
  float* part;     // partial slots, G * (D + 2) floats each: m[G], l[G], o[G][D]
  int* err;        // workspace error word
  int64_t n_tiles_total;  // NT
  int64_t wait_limit_ns;
  int32_t grid;           // P
  int32_t batch;
  int32_t n_kv_heads;
  int32_t n_q_heads;
  float scale_log2;       // scale * log2(e): scores come out in base-2 units
  int32_t debug_skip_tile;
  int32_t unit_aligned;   // 1: CTA ranges start at unit boundaries, so no unit is shared by CTAs
  // Several query tokens per sequence: q is [B][n_queries][Hq][D] (out and lse alike) and the
  // G rows of a unit are query tokens q_first + r / heads, query heads h * heads + r % heads,
  // heads = 1 << log2_heads; query token j sees the first S - n_queries + j + 1 keys.  Plain
  // decode: n_queries = 1, q_first = 0, heads = G.
  int32_t n_queries;
  int32_t q_first;
  int32_t log2_heads;
  // Paged cache (block_table != nullptr): k and v are [num_pages][Hkv][page_size][D]; sequence
  // b's logical block i (tokens i * page_size ...) is physical block block_table[b * bt_stride + i].
  // kv_off is unused then.
  const int32_t* block_table;  // this launch's first sequence's row
  int64_t bt_stride;
  int64_t num_pages;
  int32_t log2_page;
  // Shared-prefix decode (bifurcated summary: the two parts' statistics merge exactly): the
  // prefix pass's chunk statistics, folded into every row before it is written (nullptr: none).
  // Row (sequence b of this launch, head g of KV head h) has pre_chunks entries at
  // pre_part + ((c * n_kv_heads + h) * pre_rows + b * heads + g) * pre_stride, each m (log2
  // units), l, two spare floats, o[D]; the pointer already skips the launch's earlier rows.
  const float* pre_part;
  int32_t pre_chunks;
  int32_t pre_rows;
  int32_t pre_stride;
  int64_t kv_off[kMaxSeqPerLaunch];
  int64_t seq_len[kMaxSeqPerLaunch];
  int64_t tile_off[kMaxSeqPerLaunch + 1];  // first tile of sequence b on the line
  int32_t n_tiles[kMaxSeqPerLaunch];       // tiles per (sequence, KV head), >= 1
};
static_assert(sizeof(SplitParams) <= 4096, "kernel parameters must fit the 4 KB parameter space");

// Tile configurations of the split kernel (measured on B200; see the design notes).
// LongTiles: 12 consumer warps, 8 row elements per lane, 48 KB K and V tiles, a 2-deep ring:
// long sequences stream at the HBM roofline.  ShortTiles: 8 warps, 8 elements per lane,
// 16 KB tiles (64 tokens at D = 128), a 4-deep ring: short sequences waste less of their
// last tile.
struct LongTiles {
  static constexpr int warps = 12, stages = 2, elems = 8, tile_bytes = 49152;
};
struct ShortTiles {
  static constexpr int warps = 8, stages = 4, elems = 8, tile_bytes = 16384;
};

constexpr int kSmemLimit = 232448;  // opt-in shared memory per CTA on sm_100 (227 KB)

template <typename T, int D_, int G_, class V = LongTiles>
struct SplitCfg {
  static constexpr int D = D_;
  static constexpr int G = G_;
  static constexpr int ELEM = sizeof(T);
  static constexpr int EPC = 16 / ELEM;        // elements per 16-byte chunk
  // Row elements held by one lane (at least one chunk; G = 8 halves it to bound registers).
  static constexpr int E = (G >= 8) ? (V::elems / 2 > EPC ? V::elems / 2 : EPC) : V::elems;
  static constexpr int E2 = E / 2;             // ... as float pairs (packed FP32 math)
  static constexpr int LPT = D / E;            // lanes per token
  static constexpr int TPW = 32 / LPT;         // tokens per warp step
  static constexpr int ROW = D * ELEM;         // bytes per token row
  // G = 8 keeps at most 8 consumer warps: its q and o registers need more than the 128 per
  // thread that 13 resident warps leave (4 warps on one SM sub-partition).
  static constexpr int NCW = (G >= 8 && V::warps > 8) ? 8 : V::warps;  // consumer warps
  static constexpr int NSTAGE = V::stages;
  static constexpr int MERGE_BATCH = 128;      // partials whose weights are staged at once
  // Shared memory besides the ring: per-warp statistics, merge weights, barriers and flags.
  static constexpr int FIXED_SMEM =
      NCW * G * D * 4 + 2 * NCW * G * 4 + MERGE_BATCH * G * 4 + NSTAGE * G * D * ELEM + 1024;
  static constexpr int MAX_TILE_BYTES = (kSmemLimit - FIXED_SMEM) / (2 * NSTAGE);
  static constexpr int TILE_TARGET = V::tile_bytes < MAX_TILE_BYTES ? V::tile_bytes : MAX_TILE_BYTES;
  static constexpr int STEPS_FIT = TILE_TARGET / (ROW * NCW * TPW);
  // Tokens per warp per tile (phase length).  Longer phases give more independent work per
  // warp but hold more registers: 8 (4 when G = 8, whose q and o take twice the registers).
  static constexpr int MAX_STEPS = G >= 8 ? 4 : 8;
  static constexpr int STEPS = STEPS_FIT < 1 ? 1 : (STEPS_FIT > MAX_STEPS ? MAX_STEPS : STEPS_FIT);
  static constexpr int TILE = NCW * STEPS * TPW;  // tokens per tile
  static constexpr int PPC = EPC / 2;          // float pairs per chunk
  static constexpr int NCH = E / EPC;          // chunks per lane per row
  static constexpr int TILE_BYTES = TILE * ROW;
  static constexpr int NCT = NCW * 32;         // consumer threads
  static constexpr int THREADS = NCT + 32;     // + one producer warp
  static constexpr int SLOT = G * (D + 2);     // floats per partial slot
  static constexpr int NCOL = (G * D + NCT - 1) / NCT;
  static_assert(G <= LPT, "each lane must end with one head's score");
  static_assert(NCW >= G, "the merge uses one warp per head");
  static_assert(NCH >= 1 && NCH <= 4, "chunk rotation covers 1, 2 or 4 chunks");
};

template <class C>
struct SplitSmem {
  alignas(128) uint8_t k[C::NSTAGE][C::TILE_BYTES];
  alignas(128) uint8_t v[C::NSTAGE][C::TILE_BYTES];
  alignas(16) uint8_t q[C::NSTAGE][C::G * C::D * C::ELEM];  // q of a unit, copied with its first tile
  float wo[C::NCW][C::G][C::D];  // per-warp statistics of the current unit
  float wm[C::NCW][C::G];
  float wl[C::NCW][C::G];
  float mw[C::MERGE_BATCH][C::G];  // merge weights 2^(m_c - M)
  float mM[C::G];
  float mL[C::G];
  uint64_t full[C::NSTAGE];   // K and V (and q with a unit's first tile) of the stage landed
  uint64_t empty[C::NSTAGE];
  int is_last;
  int abort;
};

// ---------------------------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------------------------

// Head held by lane `li` of a token group after reduce_scores (see there).
template <int G, int LPT>
__device__ __forceinline__ int head_of_lane(int li) {
  int h = 0;
#pragma unroll
  for (int half = G >> 1, off = LPT >> 1; half >= 1; half >>= 1, off >>= 1)
    if (li & off) h += half;
  return h;
}

template <int G, int LPT>
__device__ __forceinline__ int lane_of_head(int g) {
  int li = 0;
#pragma unroll
  for (int half = G >> 1, off = LPT >> 1; half >= 1; half >>= 1, off >>= 1)
    if (g & half) li += off;
  return li;
}

// Sum G per-lane partial dot products over the LPT lanes of a token group.  While
// more than one head is left, each exchange halves the heads a lane carries (the
// lane keeps the half selected by its lane bit and receives its partner's share of
// it); the remaining exchanges are plain butterflies.  Afterwards the lane holds
// the full score of head head_of_lane(li); lanes holding the same head agree bit
// for bit (a + b == b + a).
template <int G, int LPT>
__device__ __forceinline__ float reduce_scores(float (&v)[G], int li) {
  int n = G;
#pragma unroll
  for (int off = LPT >> 1; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (li & off) != 0;
#pragma unroll
      for (int j = 0; j < G / 2; ++j) {
        if (j < n / 2) {
          const float send = upper ? v[j] : v[j + n / 2];
          const float keep = upper ? v[j + n / 2] : v[j];
          v[j] = keep + __shfl_xor_sync(kFull, send, off);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(kFull, v[0], off);
    }
  }
  return v[0];
}

template <typename T>
struct RowLoader;

// bf16: 8 values per 16-byte chunk, widened exactly to float (bf16 is the top half of a
// float), as pairs (element 2j, element 2j+1) for packed FP32 math.
template <>
struct RowLoader<__nv_bfloat16> {
  template <int NCH>
  __device__ __forceinline__ static void load(const uint8_t* row, int li, int rot, float2* f) {
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int c = li * NCH + ((k + rot) & (NCH - 1));
      const uint4 w = *reinterpret_cast<const uint4*>(row + c * 16);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) f[k * 4 + j] = make_float2(__uint_as_float(ws[j] << 16), __uint_as_float(ws[j] & 0xffff0000u));
    }
  }
  __device__ __forceinline__ static float scalar(const void* base, int64_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  }
};

template <>
struct RowLoader<float> {
  template <int NCH>
  __device__ __forceinline__ static void load(const uint8_t* row, int li, int rot, float2* f) {
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int c = li * NCH + ((k + rot) & (NCH - 1));
      const float4 w = *reinterpret_cast<const float4*>(row + c * 16);
      f[k * 2 + 0] = make_float2(w.x, w.y);
      f[k * 2 + 1] = make_float2(w.z, w.w);
    }
  }
  __device__ __forceinline__ static float scalar(const void* base, int64_t i) {
    return reinterpret_cast<const float*>(base)[i];
  }
};

// A lane reads its NCH chunks of a row starting at chunk `rot` (bank-conflict avoidance),
// so register pair j holds chunk (j / PPC + rot) mod NCH of the lane's slice.  This puts
// the pairs back in column order (pair j = columns li*E + 2j, +1) so that lanes of
// different token groups, whose rotations differ, can be added register by register.
template <int NCH, int PPC>
__device__ __forceinline__ void unrotate(float2 (&a)[NCH * PPC], int rot) {
  if constexpr (NCH > 1) {
    float2 t[NCH * PPC];
#pragma unroll
    for (int c = 0; c < NCH; ++c)
#pragma unroll
      for (int j = 0; j < PPC; ++j) {
        float2 v = a[c * PPC + j];
#pragma unroll
        for (int r = 1; r < NCH; ++r)
          if (rot == r) v = a[((c - r + NCH) % NCH) * PPC + j];
        t[c * PPC + j] = v;
      }
#pragma unroll
    for (int i = 0; i < NCH * PPC; ++i) a[i] = t[i];
  }
}

// Walks the tile line: unit (b, h), tile j of that unit.
struct TileWalk {
  int b, h;
  int64_t j;
  __device__ __forceinline__ void init(const SplitParams& p, int64_t t) {
    int lo = 0, hi = p.batch - 1;  // last b with tile_off[b] <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.tile_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    b = lo;
    const int64_t r = t - p.tile_off[b];
    h = static_cast<int>(r / p.n_tiles[b]);
    j = r % p.n_tiles[b];
  }
  __device__ __forceinline__ void next(const SplitParams& p) {
    if (++j == p.n_tiles[b]) {
      j = 0;
      if (++h == p.n_kv_heads) {
        h = 0;
        ++b;
      }
    }
  }
};

__device__ __forceinline__ int cta_of_tile(int64_t t, int64_t NT, int P) {
  return static_cast<int>(((t + 1) * P - 1) / NT);
}

// First tile of CTA i: i*NT/P, rounded up to the next (sequence, KV head) unit start when the
// plan keeps units whole.
__device__ __forceinline__ int64_t cta_first_tile(const SplitParams& p, int i) {
  const int64_t NT = p.n_tiles_total;
  const int64_t t = static_cast<int64_t>(i) * NT / p.grid;
  if (!p.unit_aligned || t >= NT) return t;
  TileWalk w;
  w.init(p, t);
  return w.j == 0 ? t : t - w.j + p.n_tiles[w.b];
}

// Sum of leaves in a fixed pairwise tree: leaf n is combined with the pending
// subtrees as a binary counter carries, so the shape depends only on the leaf count.
struct PairwiseSum {
  float s[24];
  int n = 0;
  int top = 0;
  __device__ __forceinline__ void push(float x) {
    for (int c = n; c & 1; c >>= 1) x = s[--top] + x;
    s[top++] = x;
    ++n;
  }
  __device__ __forceinline__ float result() const {
    if (top == 0) return 0.f;
    float r = s[top - 1];
    for (int j = top - 2; j >= 0; --j) r = s[j] + r;
    return r;
  }
};

// Pairwise sum of a[OFF .. OFF+N) in a fixed balanced tree.
template <int N, int OFF = 0, int M>
__device__ __forceinline__ float tree_sum(const float (&a)[M]) {
  if constexpr (N == 1) {
    return a[OFF];
  } else {
    return tree_sum<N / 2, OFF>(a) + tree_sum<N - N / 2, OFF + N / 2>(a);
  }
}

// out = O / L, lse = ln(2) (M + log2 L); an empty unit gives 0 and -inf; a unit whose
// inputs may be incomplete (this CTA gave up waiting: `poisoned`) gives NaN.  NaN partials
// of another CTA propagate through the merge weights (2^(NaN - M) is NaN).
__device__ __forceinline__ void write_final(const SplitParams& p, int b, int h, int r, int d, int D, float M,
                                            float L, float O, bool write_lse, bool poisoned) {
  if (p.pre_part != nullptr) {
    // The prefix chunks of this row, in chunk order: M' = max(M, m_c); L and O rescaled to M'.
    const int64_t cstride = static_cast<int64_t>(p.n_kv_heads) * p.pre_rows * p.pre_stride;
    const float* base =
        p.pre_part + (static_cast<int64_t>(h) * p.pre_rows + (b << p.log2_heads) + r) * p.pre_stride;
    float Mx = M;
#pragma unroll 6
    for (int c = 0; c < p.pre_chunks; ++c) Mx = fmaxf(Mx, base[c * cstride]);
    const float a = (M == -INFINITY) ? 0.f : ex2(M - Mx);
    L *= a;
    O *= a;
#pragma unroll 6
    for (int c = 0; c < p.pre_chunks; ++c) {
      const float* pc = base + c * cstride;
      const float mc = pc[0];
      const float w = (mc == -INFINITY) ? 0.f : ex2(mc - Mx);
      L += w * pc[1];
      O += w * pc[4 + d];
    }
    M = Mx;
    // a prefix CTA that gave up left an empty partial and set the error word
    poisoned = poisoned || *reinterpret_cast<const volatile int*>(p.err) != 0;
  }
  float ov, lv;
  if (L > 0.f) {
    ov = O / L;
    lv = (M + log2f(L)) * kLn2;
  } else {
    ov = 0.f;
    lv = -INFINITY;
  }
  if (poisoned || L != L) {
    ov = __int_as_float(0x7fc00000);
    lv = ov;
  }
  const int64_t row = (static_cast<int64_t>(b) * p.n_queries + p.q_first + (r >> p.log2_heads)) * p.n_q_heads +
                      (h << p.log2_heads) + (r & ((1 << p.log2_heads) - 1));
  p.out[row * D + d] = ov;
  if (write_lse) p.lse[row] = lv;
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------

// PAGED: the cache is read through p.block_table (a separate instance, so the contiguous
// kernels carry none of the paged producer's code).
template <typename T, int D, int G, class V, bool PAGED = false>
__global__ void __launch_bounds__(SplitCfg<T, D, G, V>::THREADS, 1)
    split_kv_decode_kernel(const __grid_constant__ SplitParams p) {
  using C = SplitCfg<T, D, G, V>;
  constexpr int E2 = C::E2;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SplitSmem<C>& sm = *reinterpret_cast<SplitSmem<C>*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int cta = blockIdx.x;
  const int64_t NT = p.n_tiles_total;
  const int64_t t_lo = cta_first_tile(p, cta);
  const int64_t t_hi = cta_first_tile(p, cta + 1);
  const int n_my = static_cast<int>(t_hi - t_lo);

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], C::NCW);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort;

  if (warp == C::NCW) {
    // ------------------------------- producer -------------------------------
    const uint64_t pol = l2_policy_evict_first();
    TileWalk w;
    w.init(p, t_lo);
    int fills[C::NSTAGE];
#pragma unroll
    for (int st = 0; st < C::NSTAGE; ++st) fills[st] = 0;
    if constexpr (!PAGED) {
      // Contiguous cache: lane 0 alone waits for each stage and issues at once (the ring is
      // only NSTAGE deep, so any delay between "stage free" and "copies issued" is on the
      // critical path).
      if (lane == 0) {
        for (int i = 0; i < n_my; ++i) {
          const int s = i % C::NSTAGE;
          if (i >= C::NSTAGE) {
            if (!wait_phase(&sm.empty[s], ((i / C::NSTAGE) - 1) & 1, p.wait_limit_ns, abort_flag)) {
              if (!*abort_flag) atomicCAS(p.err, 0, kErrProducerWait);
              *abort_flag = 1;
            }
          }
          if (*abort_flag) break;
          const int64_t len = p.seq_len[w.b];
          const int64_t t0 = w.j * C::TILE;
          const int nv = static_cast<int>(min(static_cast<int64_t>(C::TILE), len - t0));
          if (!(cta == 0 && i == p.debug_skip_tile)) {
            const uint32_t bytes = static_cast<uint32_t>(nv) * C::ROW;
            constexpr uint32_t q_bytes = G * D * C::ELEM;
            const bool with_q = (i == 0 || w.j == 0);  // the consumers switch to this unit here
            mbar_arrive_expect_tx(&sm.full[s], 2 * bytes + (with_q ? q_bytes : 0));
            if (with_q) {
              // One copy per query token of the launch: its `heads` query heads are contiguous.
              const int heads = 1 << p.log2_heads;
              const uint32_t qb = static_cast<uint32_t>(heads) * D * C::ELEM;
              for (int jl = 0; jl < (G >> p.log2_heads); ++jl) {
                const uint8_t* qsrc =
                    reinterpret_cast<const uint8_t*>(p.q) +
                    ((static_cast<int64_t>(w.b) * p.n_queries + p.q_first + jl) * p.n_q_heads + w.h * heads) * D *
                        C::ELEM;
                bulk_load(sm.q[s] + jl * qb, qsrc, qb, &sm.full[s], pol);
              }
            }
            if (bytes != 0) {
              const int64_t off = p.kv_off[w.b] + (static_cast<int64_t>(w.h) * len + t0) * D;
              bulk_load(sm.k[s], reinterpret_cast<const T*>(p.k) + off, bytes, &sm.full[s], pol);
              bulk_load(sm.v[s], reinterpret_cast<const T*>(p.v) + off, bytes, &sm.full[s], pol);
            }
            ++fills[s];
          }
          w.next(p);
        }
      }
    } else {
      // Stage s's expected bytes and the unit's q, which lands with the unit's first tile (one
      // copy per query token of the launch: its `heads` query heads are contiguous).  Lane 0.
      auto tile_header = [&](int s, int i, uint32_t bytes) {
        constexpr uint32_t q_bytes = G * D * C::ELEM;
        const bool with_q = (i == 0 || w.j == 0);  // the consumers switch to this unit here
        mbar_arrive_expect_tx(&sm.full[s], 2 * bytes + (with_q ? q_bytes : 0));
        if (with_q) {
          const int heads = 1 << p.log2_heads;
          const uint32_t qb = static_cast<uint32_t>(heads) * D * C::ELEM;
          for (int jl = 0; jl < (G >> p.log2_heads); ++jl) {
            const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q) +
                                  ((static_cast<int64_t>(w.b) * p.n_queries + p.q_first + jl) * p.n_q_heads +
                                   w.h * heads) * D * C::ELEM;
            bulk_load(sm.q[s] + jl * qb, qsrc, qb, &sm.full[s], pol);
          }
        }
      };
      auto stage_wait = [&](int s, int i) {  // lane 0: the stage's previous tile was consumed
        if (i >= C::NSTAGE && !wait_phase(&sm.empty[s], ((i / C::NSTAGE) - 1) & 1, p.wait_limit_ns, abort_flag)) {
          if (!*abort_flag) atomicCAS(p.err, 0, kErrProducerWait);
          *abort_flag = 1;
        }
      };
      // Paged cache: one copy per page a tile touches, lane k taking page k (at most 25 pages:
      // 384-token tiles of 16-token pages).  Each lane loads its block-table entry one tile
      // ahead; the warp checks a tile's entries against num_pages before anything is expected
      // on the stage's barrier, so nothing is ever read through a bad entry.
      auto fetch = [&](const TileWalk& tw, int64_t* page, int* n_pg, bool* bad) {
        const int64_t len = p.seq_len[tw.b];
        const int64_t t0 = tw.j * C::TILE;
        const int64_t nv = min(static_cast<int64_t>(C::TILE), len - t0);
        *page = 0;
        *n_pg = 0;
        *bad = false;
        if (nv > 0) {
          const int64_t pg0 = t0 >> p.log2_page;
          *n_pg = static_cast<int>(((t0 + nv - 1) >> p.log2_page) - pg0 + 1);
          if (lane < *n_pg) {
            *page = __ldg(p.block_table + tw.b * p.bt_stride + pg0 + lane);
            *bad = *page < 0 || *page >= p.num_pages;
          }
        }
      };
      int64_t page = 0;
      int n_pg = 0;
      bool bad = false;
      if (n_my > 0) fetch(w, &page, &n_pg, &bad);
      for (int i = 0; i < n_my; ++i) {
        const int s = i % C::NSTAGE;
        int64_t page_n = 0;
        int n_pg_n = 0;
        bool bad_n = false;
        if (i + 1 < n_my) {
          TileWalk wn = w;
          wn.next(p);
          fetch(wn, &page_n, &n_pg_n, &bad_n);
        }
        if (lane == 0) stage_wait(s, i);
        if (__any_sync(kFull, bad)) {
          if (lane == 0) {
            atomicCAS(p.err, 0, kErrBadPage);
            *abort_flag = 1;
          }
          break;
        }
        const int64_t len = p.seq_len[w.b];
        const int64_t t0 = w.j * C::TILE;
        const int nv = static_cast<int>(min(static_cast<int64_t>(C::TILE), len - t0));
        const bool skip = (cta == 0 && i == p.debug_skip_tile);
        bool go = false;
        if (lane == 0) {
          go = *abort_flag == 0;
          if (go && !skip) {
            tile_header(s, i, static_cast<uint32_t>(nv) * C::ROW);
            ++fills[s];
          }
        }
        if (!__shfl_sync(kFull, go, 0)) break;
        if (!skip && lane < n_pg) {
          const int64_t ps = int64_t(1) << p.log2_page;
          const int64_t first = ((t0 >> p.log2_page) + lane) << p.log2_page;  // first token of the page
          const int64_t lo = max(t0, first), hi = min(t0 + nv, first + ps);
          const uint32_t nb = static_cast<uint32_t>(hi - lo) * C::ROW;
          const int64_t row = ((page * p.n_kv_heads + w.h) << p.log2_page) + (lo - first);
          bulk_load(sm.k[s] + (lo - t0) * C::ROW, reinterpret_cast<const T*>(p.k) + row * D, nb, &sm.full[s], pol);
          bulk_load(sm.v[s] + (lo - t0) * C::ROW, reinterpret_cast<const T*>(p.v) + row * D, nb, &sm.full[s], pol);
        }
        page = page_n;
        n_pg = n_pg_n;
        bad = bad_n;
        w.next(p);
      }
    }
    // No copy may still be landing in shared memory when the CTA exits.
    if (lane == 0) {
#pragma unroll
      for (int st = 0; st < C::NSTAGE; ++st) {
        if (fills[st] > 0 && !wait_phase(&sm.full[st], (fills[st] - 1) & 1, p.wait_limit_ns, nullptr))
          atomicCAS(p.err, 0, kErrDrainWait);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------- consumers ------------------------------
    // Lane layout: token group gi (one token per group per step) of LPT lanes; lane li of
    // a group holds E columns of the row (its NCH chunks, read from chunk `rot` on).
    const int li = lane % C::LPT;
    const int gi = lane / C::LPT;
    const int rot = (lane / (8 / C::NCH)) % C::NCH;
    int src_lane[G];
#pragma unroll
    for (int g = 0; g < G; ++g) src_lane[g] = gi * C::LPT + lane_of_head<G, C::LPT>(g);
    auto dcol = [&](int e) {  // column of register element e (load order)
      const int c = li * C::NCH + (((e / C::EPC) + rot) & (C::NCH - 1));
      return c * C::EPC + e % C::EPC;
    };

    float2 q2[G][E2];  // q * scale * log2(e), the G heads of the current KV head
    float2 o2[G][E2];  // unnormalised output of this lane's tokens
    float m = -INFINITY, l = 0.f;  // statistics of head head_of_lane(li) over this lane's tokens
    // Keys at the end of the sequence this lane's row may not see: query token j of n is
    // n - 1 - j positions before the last one (0 for plain decode).
    const int lag = p.n_queries - 1 - (p.q_first + (head_of_lane<G, C::LPT>(li) >> p.log2_heads));

    // The unit's q (landed in stage s with the unit's first tile), read like a K row so the
    // register order matches the K elements it multiplies.
    auto load_q = [&](int s) {
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        RowLoader<T>::template load<C::NCH>(sm.q[s] + g * C::ROW, li, rot, q2[g]);
#pragma unroll
        for (int j = 0; j < E2; ++j) q2[g][j] = __fmul2_rn(q2[g][j], sc2);
      }
    };
    auto reset = [&]() {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < E2; ++j) o2[g][j] = make_float2(0.f, 0.f);
      m = -INFINITY;
      l = 0.f;
    };

    // Combine the statistics of every consumer lane for unit (b, h) and emit them.
    auto finalize = [&](int b, int h) {
      // 1) merge the TPW token groups of this warp (butterflies across groups)
#pragma unroll
      for (int g = 0; g < G; ++g) unrotate<C::NCH, C::PPC>(o2[g], rot);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mg = __shfl_sync(kFull, m, src_lane[g]);
        const float lg = __shfl_sync(kFull, l, src_lane[g]);
        float Mx = mg;
#pragma unroll
        for (int off = C::LPT; off < 32; off <<= 1) Mx = fmaxf(Mx, __shfl_xor_sync(kFull, Mx, off));
        const float a = (mg == -INFINITY) ? 0.f : ex2(mg - Mx);
        float ls = lg * a;
#pragma unroll
        for (int j = 0; j < E2; ++j) o2[g][j] = __fmul2_rn(o2[g][j], make_float2(a, a));
#pragma unroll
        for (int off = C::LPT; off < 32; off <<= 1) {
          ls += __shfl_xor_sync(kFull, ls, off);
#pragma unroll
          for (int j = 0; j < E2; ++j) {
            o2[g][j].x += __shfl_xor_sync(kFull, o2[g][j].x, off);
            o2[g][j].y += __shfl_xor_sync(kFull, o2[g][j].y, off);
          }
        }
        if (lane == 0) {
          sm.wm[warp][g] = Mx;
          sm.wl[warp][g] = ls;
        }
        if (gi == 0) {
#pragma unroll
          for (int j = 0; j < E2; ++j) {
            sm.wo[warp][g][li * C::E + 2 * j] = o2[g][j].x;
            sm.wo[warp][g][li * C::E + 2 * j + 1] = o2[g][j].y;
          }
        }
      }
      named_barrier(1, C::NCT);

      // 2) merge the warps; write the final result or this CTA's partial
      const bool poisoned = *abort_flag != 0;
      const int unit = b * p.n_kv_heads + h;
      const int64_t U0 = p.tile_off[b] + static_cast<int64_t>(h) * p.n_tiles[b];
      const int i_first = cta_of_tile(U0, NT, p.grid);
      const int i_last = cta_of_tile(U0 + p.n_tiles[b] - 1, NT, p.grid);
      const int n_parts = p.unit_aligned ? 1 : i_last - i_first + 1;
      float* slot = p.part + static_cast<int64_t>(cta + unit) * C::SLOT;
#pragma unroll
      for (int k = 0; k < C::NCOL; ++k) {
        const int col = tid + k * C::NCT;
        if (col < G * D) {
          const int g = col / D, d = col % D;
          float Mx = -INFINITY;
#pragma unroll
          for (int w = 0; w < C::NCW; ++w) Mx = fmaxf(Mx, sm.wm[w][g]);
          float ao[C::NCW], al[C::NCW];
#pragma unroll
          for (int w = 0; w < C::NCW; ++w) {
            const float mw = sm.wm[w][g];
            const float a = (mw == -INFINITY) ? 0.f : ex2(mw - Mx);
            ao[w] = a * sm.wo[w][g][d];
            al[w] = a * sm.wl[w][g];
          }
          const float O = tree_sum<C::NCW>(ao), L = tree_sum<C::NCW>(al);
          if (n_parts == 1) {
            write_final(p, b, h, g, d, D, Mx, L, O, d == 0, poisoned);
          } else {
            const float nan = __int_as_float(0x7fc00000);
            slot[2 * G + g * D + d] = poisoned ? nan : O;
            if (d == 0) {
              slot[g] = poisoned ? nan : Mx;
              slot[G + g] = poisoned ? nan : L;
            }
          }
        }
      }
      if (n_parts > 1) {
        __threadfence();
        named_barrier(1, C::NCT);
        if (tid == 0) sm.is_last = (atomicAdd(&p.tickets[unit], 1) == n_parts - 1);
        named_barrier(1, C::NCT);
        if (sm.is_last) {
          // 3) last CTA of the unit: a tree over the unit's partials fixed by their count
          __threadfence();
          const float* base = p.part + static_cast<int64_t>(i_first + unit) * C::SLOT;
          const int n = n_parts;
          if (warp < G) {
            float Mx = -INFINITY;
            for (int c = lane; c < n; c += 32) Mx = fmaxf(Mx, ld_cg(base + static_cast<int64_t>(c) * C::SLOT + warp));
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) Mx = fmaxf(Mx, __shfl_xor_sync(kFull, Mx, off));
            if (lane == 0) sm.mM[warp] = Mx;
          }
          named_barrier(1, C::NCT);
          PairwiseSum acc[C::NCOL], accl[C::NCOL];
          for (int c0 = 0; c0 < n; c0 += C::MERGE_BATCH) {
            const int nb = min(C::MERGE_BATCH, n - c0);
            for (int idx = tid; idx < nb * G; idx += C::NCT) {
              const int c = idx / G, g = idx % G;
              const float mv = ld_cg(base + static_cast<int64_t>(c0 + c) * C::SLOT + g);
              sm.mw[c][g] = (mv == -INFINITY) ? 0.f : ex2(mv - sm.mM[g]);
            }
            named_barrier(1, C::NCT);
#pragma unroll
            for (int k = 0; k < C::NCOL; ++k) {
              const int col = tid + k * C::NCT;
              if (col < G * D) {
                const int g = col / D, d = col % D;
                // Leaves in batches of 16: the batch's loads are in flight together; each batch
                // is summed by a fixed balanced tree (in registers) and its sum enters the
                // pairwise sum in order, one push per batch (the pairwise state is indexed at run
                // time and lives in local memory).
                constexpr int LB = 16;
                for (int cb = 0; cb < nb; cb += LB) {
                  float ov[LB], lv[LB];
#pragma unroll
                  for (int u = 0; u < LB; ++u) {
                    const bool in = cb + u < nb;
                    const float* sp = base + static_cast<int64_t>(c0 + cb + u) * C::SLOT;
                    ov[u] = in ? ld_cg(sp + 2 * G + g * D + d) : 0.f;
                    lv[u] = (in && d == 0) ? ld_cg(sp + G + g) : 0.f;
                  }
#pragma unroll
                  for (int u = 0; u < LB; ++u) {
                    const float wgt = (cb + u < nb) ? sm.mw[cb + u][g] : 0.f;
                    ov[u] *= wgt;
                    lv[u] *= wgt;
                  }
                  acc[k].push(tree_sum<LB>(ov));
                  if (d == 0) accl[k].push(tree_sum<LB>(lv));
                }
              }
            }
            named_barrier(1, C::NCT);
          }
#pragma unroll
          for (int k = 0; k < C::NCOL; ++k) {
            const int col = tid + k * C::NCT;
            if (col < G * D && col % D == 0) sm.mL[col / D] = accl[k].result();
          }
          named_barrier(1, C::NCT);
#pragma unroll
          for (int k = 0; k < C::NCOL; ++k) {
            const int col = tid + k * C::NCT;
            if (col < G * D) {
              const int g = col / D, d = col % D;
              write_final(p, b, h, g, d, D, sm.mM[g], sm.mL[g], acc[k].result(), d == 0, poisoned);
            }
          }
          if (tid == 0) p.tickets[unit] = 0;
        }
      }
      named_barrier(1, C::NCT);
    };

    TileWalk w;
    w.init(p, t_lo);
    int cur_b = w.b, cur_h = w.h;
    reset();
    bool new_unit = true;

    for (int i = 0; i < n_my; ++i) {
      if (w.b != cur_b || w.h != cur_h) {
        finalize(cur_b, cur_h);
        cur_b = w.b;
        cur_h = w.h;
        reset();
        new_unit = true;
      }
      const int s = i % C::NSTAGE;
      bool ok = (*abort_flag == 0);
      if (ok) ok = wait_phase(&sm.full[s], (i / C::NSTAGE) & 1, p.wait_limit_ns, abort_flag);
      ok = __all_sync(kFull, ok);
      if (!ok && lane == 0) {
        if (!*abort_flag) atomicCAS(p.err, 0, kErrConsumerWait);
        *abort_flag = 1;
      }
      if (ok && new_unit) {
        load_q(s);
        new_unit = false;
      }
      if (ok) {
        const int64_t len = p.seq_len[w.b];
        const int nv = static_cast<int>(min(static_cast<int64_t>(C::TILE), len - w.j * C::TILE));
        const int nv_row = static_cast<int>(min(static_cast<int64_t>(C::TILE), len - lag - w.j * C::TILE));
        const uint8_t* kt = sm.k[s];
        const uint8_t* vt = sm.v[s];
        // Phase A: the scores of this warp's STEPS tokens of the tile (independent chains).
        float x[C::STEPS];
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
          const int tok = (warp * C::STEPS + st) * C::TPW + gi;
          float2 kf[E2];
          RowLoader<T>::template load<C::NCH>(kt + tok * C::ROW, li, rot, kf);
          float sc[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < E2; ++j) acc = __ffma2_rn(q2[g][j], kf[j], acc);
            sc[g] = acc.x + acc.y;
          }
          const float xs = reduce_scores<G, C::LPT>(sc, li);
          x[st] = (tok < nv_row) ? xs : -INFINITY;
        }
        // Phase B: one online-softmax update for the tile (lazy rescaling of m).
        float xm = x[0];
#pragma unroll
        for (int st = 1; st < C::STEPS; ++st) xm = fmaxf(xm, x[st]);
        const bool need = xm > m + kRescaleThreshold;
        if (__any_sync(kFull, need)) {
          const float mn = need ? xm : m;
          const float a = need ? ex2(m - mn) : 1.f;
          l *= a;
          m = mn;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float ag = __shfl_sync(kFull, a, src_lane[g]);
#pragma unroll
            for (int j = 0; j < E2; ++j) o2[g][j] = __fmul2_rn(o2[g][j], make_float2(ag, ag));
          }
        }
        float pe[C::STEPS];
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
          pe[st] = (x[st] == -INFINITY) ? 0.f : ex2(x[st] - m);
          l += pe[st];
        }
        // Phase C: o += p v for the same tokens.
#pragma unroll
        for (int st = 0; st < C::STEPS; ++st) {
          const int tok = (warp * C::STEPS + st) * C::TPW + gi;
          float pg[G];
#pragma unroll
          for (int g = 0; g < G; ++g) pg[g] = __shfl_sync(kFull, pe[st], src_lane[g]);
          if (ok && tok < nv) {
            float2 vf[E2];
            RowLoader<T>::template load<C::NCH>(vt + tok * C::ROW, li, rot, vf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float2 pp = make_float2(pg[g], pg[g]);
#pragma unroll
              for (int j = 0; j < E2; ++j) o2[g][j] = __ffma2_rn(pp, vf[j], o2[g][j]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      w.next(p);
    }
    if (n_my > 0) finalize(cur_b, cur_h);
  }
  __syncthreads();
}

}  // namespace ta
