// Decode over many short (sequence, KV head) units.  It serves the suffix part of shared-prefix
// decode (Bifurcated attention summary, briefgpt.xyz, 2403.08845, TL;DR: the per-sample decoded
// tokens are a second, separate product): hundreds of units of a few hundred tokens each, whose
// K/V are read once.  The result folds in the prefix pass's chunk statistics before it is
// written (their exact merge: max and logsumexp are associative, Tree Attention article,
// m.srwj168.com.cn, "The energy view of attention").
//
// Persistent CTAs (two per SM, one for G = 8) take units u = blockIdx.x, blockIdx.x + gridDim.x,
// ...  Warp 0's first lane streams every unit's keys, 32 at a time, into a ring of shared-memory
// stages with 1-D bulk copies (K rows, V rows and the unit's G query rows per stage), so the ring
// keeps loading across unit boundaries; the eight other warps take a unit's stages round robin,
// each with its own online-softmax state (the "Attention acceleration" concept page,
// compassingai.com, Technical principles 2.1, in base 2, O kept unnormalised).  Per stage and
// warp:
//   scores:  lane l owns columns 4l .. 4l + 3 of q and of every K row; the 32 partial sums of
//            32 / G keys x G heads are reduced across the lanes in one transposed butterfly
//            (31 shuffles), after which lane i holds key i / G, head i % G;
//   softmax: the stage max per head (shuffles), lazy rescale when it exceeds the running max by
//            more than 8 (exact: l and o share the reference);
//   p V:     lane l accumulates columns 4l .. 4l + 3 of every head (packed FMAs); the stage's
//            weights pass through shared memory, one broadcast read per key.
// No warp waits for another: at a unit's end each warp folds its share of the prefix chunks'
// statistics (chunks c = warp, warp + 8, ...) into its own (m, l, o), writes that partial to one
// of two shared buffers, and the last warp to arrive merges the eight partials in a fixed order
// and writes out = o / l and lse.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "short_decode.h"

namespace ta {
namespace {

constexpr int kD = 128;
constexpr int kKeys = 32;                // keys per stage
constexpr int kW = 8;                    // consumer warps
constexpr int kThreads = (kW + 1) * 32;  // and the loading warp
constexpr float kShortRescale = 8.0f;

template <int G>
struct ShortCfg {
  static constexpr int kCtasPerSm = G == 8 ? 1 : 2;
  static constexpr int kStages = G == 8 ? 7 : 4;
  static constexpr int kKvBytes = kKeys * kD * 2;            // K or V rows of one stage
  static constexpr int kSlotBytes = 2 * kKvBytes + G * kD * 2;  // K, V, the unit's q rows
  static constexpr int kKG = 32 / G;                         // keys per transposed reduction
};

template <int G>
struct ShortSmem {
  alignas(16) uint8_t slot[ShortCfg<G>::kStages][ShortCfg<G>::kSlotBytes];
  alignas(16) float part_o[2][kW][G][kD];  // each warp's unnormalised o of a unit (two units in turn)
  alignas(16) float pbuf[kW][kKeys * G];     // a stage's weights, [key][head]
  float part_m[2][kW][G], part_l[2][kW][G];
  uint64_t full[ShortCfg<G>::kStages], empty[ShortCfg<G>::kStages];
  int issued;     // stages the loader has issued (or skipped): a consumer tests a slot's parity only
                  // once its stage is issued, when the slot's barrier is in that stage's phase
  int ticket[2];  // warps done with the unit in partial buffer i
  int merged[2];  // units merged out of partial buffer i so far
  int abort;
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bounded wait until the loader has issued stage t.  Each slot is consumed by different warps at
// successive phases, and a parity test cannot tell a slot's next phase from the one after it: a
// warp may test stage t's phase only after stage t - R (same slot) was consumed, which the loader
// guarantees before it issues stage t.
__device__ __forceinline__ bool wait_issued(const volatile int* issued, int t, int64_t limit_ns,
                                            const volatile int* abort) {
  if (*issued > t) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(32);  // a waiting warp leaves the issue slots to the computing ones
    if (*issued > t) return true;
    if (*abort) return false;
    if (static_cast<int64_t>(global_timer_ns() - t0) > limit_ns) return false;
  }
}

// Bounded wait until *counter >= target (shared memory, written by another warp).
__device__ __forceinline__ bool wait_count(const volatile int* counter, int target, int64_t limit_ns) {
  if (*counter >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(64);
    if (*counter >= target) return true;
    if (static_cast<int64_t>(global_timer_ns() - t0) > limit_ns) return false;
  }
}

// One butterfly level: lanes with bit N set keep the upper half of v[0 .. 2N), the others the
// lower half, each adding its partner's copy of the half it keeps.
template <int N>
__device__ __forceinline__ void fold_half(float (&v)[32], int lane) {
  const bool up = (lane & N) != 0;
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const float send = up ? v[k] : v[k + N];
    const float keep = up ? v[k + N] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, N);
  }
}

// v[i] on every lane holds a partial sum of quantity i; returns the full sum of quantity `lane`.
__device__ __forceinline__ float transpose_sum(float (&v)[32], int lane) {
  fold_half<16>(v, lane);
  fold_half<8>(v, lane);
  fold_half<4>(v, lane);
  fold_half<2>(v, lane);
  fold_half<1>(v, lane);
  return v[0];
}

template <int G>
__device__ __forceinline__ void pv_key(const __nv_bfloat16* Vs, const float* pb, int j, int lane,
                                       float (&acc)[G][4]) {
  const uint2 vr = *reinterpret_cast<const uint2*>(Vs + j * kD + 4 * lane);
  const float v0 = bf_lo(vr.x), v1 = bf_hi(vr.x), v2 = bf_lo(vr.y), v3 = bf_hi(vr.y);
  float pj[G];
  if constexpr (G >= 4) {
#pragma unroll
    for (int g = 0; g < G; g += 4) {
      const float4 t = *reinterpret_cast<const float4*>(pb + j * G + g);
      pj[g] = t.x;
      pj[g + 1] = t.y;
      pj[g + 2] = t.z;
      pj[g + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int g = 0; g < G; ++g) pj[g] = pb[j * G + g];
  }
  const float2 va = make_float2(v0, v1), vb = make_float2(v2, v3);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float2 pp = make_float2(pj[g], pj[g]);
    const float2 a = __ffma2_rn(pp, va, make_float2(acc[g][0], acc[g][1]));
    const float2 c = __ffma2_rn(pp, vb, make_float2(acc[g][2], acc[g][3]));
    acc[g][0] = a.x;
    acc[g][1] = a.y;
    acc[g][2] = c.x;
    acc[g][3] = c.y;
  }
}

template <int G>
__global__ void __launch_bounds__(kThreads, ShortCfg<G>::kCtasPerSm)
    short_decode_kernel(const __grid_constant__ ShortParams p) {
  using C = ShortCfg<G>;
  constexpr int R = C::kStages;
  extern __shared__ __align__(16) uint8_t short_smem_raw[];
  ShortSmem<G>& sm = *reinterpret_cast<ShortSmem<G>*>(short_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_units = p.n_kv_heads * p.n_seq;
  volatile int* abort = &sm.abort;

  if (tid == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    sm.issued = 0;
    sm.ticket[0] = sm.ticket[1] = 0;
    sm.merged[0] = sm.merged[1] = 0;
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------ loader (one lane) ------------------------------
    if (lane != 0) return;
    const uint64_t pol = l2_policy_evict_first();
    int seq = 0;  // stages issued (or skipped by the test hook) so far
    bool ok = true;
    for (int u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
      const int b = u / p.n_kv_heads, h = u % p.n_kv_heads;
      const int64_t S = p.seq_len[b];
      const __nv_bfloat16* K = p.k + p.kv_off[b] + static_cast<int64_t>(h) * S * kD;
      const __nv_bfloat16* V = p.v + p.kv_off[b] + static_cast<int64_t>(h) * S * kD;
      const __nv_bfloat16* Q = p.q + (static_cast<int64_t>(b) * p.n_q_heads + h * G) * kD;
      const int ns = static_cast<int>((S + kKeys - 1) / kKeys);
      for (int s = 0; s < ns; ++s, ++seq) {
        const int slot = seq % R;
        if (seq >= R && !wait_phase(&sm.empty[slot], ((seq / R) - 1) & 1, p.wait_limit_ns, abort)) {
          ok = false;
          break;
        }
        if (blockIdx.x == 0 && seq + 1 == p.debug_skip_stage1) {  // never loaded
          *reinterpret_cast<volatile int*>(&sm.issued) = seq + 1;
          continue;
        }
        const uint32_t bytes = static_cast<uint32_t>(min(static_cast<int64_t>(kKeys), S - int64_t(s) * kKeys)) * kD * 2;
        uint8_t* dst = sm.slot[slot];
        mbar_arrive_expect_tx(&sm.full[slot], 2 * bytes + G * kD * 2);
        bulk_load(dst, K + static_cast<int64_t>(s) * kKeys * kD, bytes, &sm.full[slot], pol);
        bulk_load(dst + C::kKvBytes, V + static_cast<int64_t>(s) * kKeys * kD, bytes, &sm.full[slot], pol);
        bulk_load(dst + 2 * C::kKvBytes, Q, G * kD * 2, &sm.full[slot], pol);
        __threadfence_block();  // the stage's expect_tx precedes its publication
        *reinterpret_cast<volatile int*>(&sm.issued) = seq + 1;
      }
    }
    if (!ok) {
      sm.abort = 1;
      atomicCAS(p.err, 0, kErrShortWait);
    }
    // No copy may still be writing into shared memory when the CTA exits: wait (bounded) for
    // the last stage issued into each slot.
    for (int t = max(0, seq - R); t < seq; ++t) {
      if (blockIdx.x == 0 && t + 1 == p.debug_skip_stage1) continue;
      if (!wait_phase(&sm.full[t % R], (t / R) & 1, p.wait_limit_ns, nullptr)) atomicCAS(p.err, 0, kErrShortWait);
    }
    return;
  }

  // ------------------------------- consumers --------------------------------------
  const int w = warp - 1;
  const float sc = p.scale_log2;
  const bool fold = p.pre_part != nullptr;
  const int nc = fold ? p.pre_chunks : 0;
  const int64_t cstride = static_cast<int64_t>(p.n_kv_heads) * p.pre_rows * p.pre_stride;
  bool ok = true;
  int seq0 = 0;  // the CTA's stage count at the start of the unit
  int ul = 0;    // the unit's index among this CTA's units
  for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++ul) {
    const int b = u / p.n_kv_heads, h = u % p.n_kv_heads;
    const int64_t S = p.seq_len[b];
    const int ns = static_cast<int>((S + kKeys - 1) / kKeys);
    float m = -INFINITY, lp = 0.f;  // head lane % G
    float acc[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;
    for (int s = w; ok && s < ns; s += kW) {
      const int t = seq0 + s, slot = t % R;
      ok = __all_sync(0xffffffffu, wait_issued(&sm.issued, t, p.wait_limit_ns, abort) &&
                                       wait_phase(&sm.full[slot], (t / R) & 1, p.wait_limit_ns, abort));
      if (!ok) break;
      const __nv_bfloat16* Ks = reinterpret_cast<const __nv_bfloat16*>(sm.slot[slot]);
      const __nv_bfloat16* Vs = Ks + kKeys * kD;
      const __nv_bfloat16* Qs = Vs + kKeys * kD;
      const int nk = static_cast<int>(min(static_cast<int64_t>(kKeys), S - int64_t(s) * kKeys));
      // q (scaled, base 2) for the lane's 4 columns, as pairs over heads (G >= 2) or columns
      float2 q2[G == 1 ? 2 : 4 * (G / 2)];
      {
        float q[G][4];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint2 qq = *reinterpret_cast<const uint2*>(Qs + g * kD + 4 * lane);
          q[g][0] = bf_lo(qq.x) * sc;
          q[g][1] = bf_hi(qq.x) * sc;
          q[g][2] = bf_lo(qq.y) * sc;
          q[g][3] = bf_hi(qq.y) * sc;
        }
        if constexpr (G == 1) {
          q2[0] = make_float2(q[0][0], q[0][1]);
          q2[1] = make_float2(q[0][2], q[0][3]);
        } else {
#pragma unroll
          for (int g2 = 0; g2 < G / 2; ++g2)
#pragma unroll
            for (int c = 0; c < 4; ++c) q2[g2 * 4 + c] = make_float2(q[2 * g2][c], q[2 * g2 + 1][c]);
        }
      }
      // scores: x[kg] = key kg * KG + lane / G, head lane % G
      float x[G];
#pragma unroll
      for (int kg = 0; kg < G; ++kg) {
        float part[32];
#pragma unroll
        for (int kk = 0; kk < C::kKG; ++kk) {
          const int key = kg * C::kKG + kk;
          const uint2 kr = key < nk ? *reinterpret_cast<const uint2*>(Ks + key * kD + 4 * lane) : make_uint2(0, 0);
          const float k0 = bf_lo(kr.x), k1 = bf_hi(kr.x), k2 = bf_lo(kr.y), k3 = bf_hi(kr.y);
          if constexpr (G == 1) {
            float2 d = __ffma2_rn(q2[0], make_float2(k0, k1), make_float2(0.f, 0.f));
            d = __ffma2_rn(q2[1], make_float2(k2, k3), d);
            part[kk] = d.x + d.y;
          } else {
#pragma unroll
            for (int g2 = 0; g2 < G / 2; ++g2) {
              float2 d = __fmul2_rn(q2[g2 * 4 + 0], make_float2(k0, k0));
              d = __ffma2_rn(q2[g2 * 4 + 1], make_float2(k1, k1), d);
              d = __ffma2_rn(q2[g2 * 4 + 2], make_float2(k2, k2), d);
              d = __ffma2_rn(q2[g2 * 4 + 3], make_float2(k3, k3), d);
              part[kk * G + 2 * g2] = d.x;
              part[kk * G + 2 * g2 + 1] = d.y;
            }
          }
        }
        const float xs = transpose_sum(part, lane);
        x[kg] = (kg * C::kKG + lane / G < nk) ? xs : -INFINITY;
      }
      // online softmax over the stage
      float cmax = x[0];
#pragma unroll
      for (int kg = 1; kg < G; ++kg) cmax = fmaxf(cmax, x[kg]);
#pragma unroll
      for (int off = G; off < 32; off <<= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
      const bool need = cmax > m + kShortRescale;
      if (__any_sync(0xffffffffu, need)) {
        const float a = need ? (m == -INFINITY ? 0.f : ex2(m - cmax)) : 1.f;
        if (need) m = cmax;
        lp *= a;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float ag = __shfl_sync(0xffffffffu, a, g);  // lane g holds head g
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[g][e] *= ag;
        }
      }
      float* pb = sm.pbuf[w];
#pragma unroll
      for (int kg = 0; kg < G; ++kg) {
        const float pk = ex2(x[kg] - m);  // 0 for keys past the stage's end
        lp += pk;
        pb[kg * 32 + lane] = pk;  // = [key][head]
      }
      __syncwarp();
      if (nk == kKeys) {
#pragma unroll 8
        for (int j = 0; j < kKeys; ++j) pv_key<G>(Vs, pb, j, lane, acc);
      } else {
        for (int j = 0; j < nk; ++j) pv_key<G>(Vs, pb, j, lane, acc);  // rows past nk were not loaded
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
    }
    if (!ok && lane == 0 && atomicExch(const_cast<int*>(abort), 1) == 0) atomicCAS(p.err, 0, kErrShortWait);
    seq0 += ns;
    // The warp's statistics per head, in every lane.
    float Mg[G], Lg[G];
    {
      float l = lp;
#pragma unroll
      for (int off = G; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        Mg[g] = __shfl_sync(0xffffffffu, m, g);
        Lg[g] = __shfl_sync(0xffffffffu, l, g);
      }
    }
    // Fold in this warp's share of the prefix chunks (their statistics exist once the prefix
    // kernel has completed).
    if (fold) {
      if (ul == 0) grid_dependency_wait();
      for (int c = w; c < nc; c += kW) {
        const float* row = p.pre_part + (static_cast<int64_t>(h) * p.pre_rows + b * G) * p.pre_stride + c * cstride;
        float mc[G], lc[G];
        float4 oc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          mc[g] = row[g * p.pre_stride];
          lc[g] = row[g * p.pre_stride + 1];
          oc[g] = *reinterpret_cast<const float4*>(row + g * p.pre_stride + 4 + 4 * lane);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float Mn = fmaxf(Mg[g], mc[g]);
          const float a = (Mg[g] == -INFINITY) ? 0.f : ex2(Mg[g] - Mn);
          const float bw = (mc[g] == -INFINITY) ? 0.f : ex2(mc[g] - Mn);
          acc[g][0] = acc[g][0] * a + oc[g].x * bw;
          acc[g][1] = acc[g][1] * a + oc[g].y * bw;
          acc[g][2] = acc[g][2] * a + oc[g].z * bw;
          acc[g][3] = acc[g][3] * a + oc[g].w * bw;
          Lg[g] = Lg[g] * a + lc[g] * bw;
          Mg[g] = Mn;
        }
      }
    }
    // The partial into buffer ul % 2, once the unit that last used it has been merged.
    const int buf = ul & 1;
    if (!wait_count(&sm.merged[buf], ul >> 1, p.wait_limit_ns)) {
      if (lane == 0 && atomicExch(const_cast<int*>(abort), 1) == 0) atomicCAS(p.err, 0, kErrShortWait);
    }
    __syncwarp();
    __threadfence_block();
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        sm.part_m[buf][w][g] = Mg[g];
        sm.part_l[buf][w][g] = Lg[g];
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
      *reinterpret_cast<float4*>(&sm.part_o[buf][w][g][4 * lane]) =
          make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&sm.ticket[buf], 1) == kW - 1;
    }
    if (!__shfl_sync(0xffffffffu, last, 0)) continue;
    // The last warp of the unit: merge the partials in warp order, write out and lse.
    __threadfence_block();
    const bool bad = *abort != 0 || (fold && *reinterpret_cast<const volatile int*>(p.err) != 0);
    const int64_t qrow0 = static_cast<int64_t>(b) * p.n_q_heads + h * G;  // the unit's first output row
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float M = -INFINITY;
#pragma unroll
      for (int v = 0; v < kW; ++v) M = fmaxf(M, sm.part_m[buf][v][g]);
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int v = 0; v < kW; ++v) {
        const float mv = sm.part_m[buf][v][g];
        const float a = (mv == -INFINITY) ? 0.f : ex2(mv - M);
        L += a * sm.part_l[buf][v][g];
        const float4 o = *reinterpret_cast<const float4*>(&sm.part_o[buf][v][g][4 * lane]);
        O = make_float4(O.x + a * o.x, O.y + a * o.y, O.z + a * o.z, O.w + a * o.w);
      }
      float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
      float lv = -INFINITY;
      if (L > 0.f) {
        const float inv = 1.f / L;
        ov = make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
        lv = (M + log2f(L)) * 0.693147180559945309f;
      }
      if (bad || L != L) {
        const float nan = __int_as_float(0x7fc00000);
        ov = make_float4(nan, nan, nan, nan);
        lv = nan;
      }
      *reinterpret_cast<float4*>(p.out + (qrow0 + g) * kD + 4 * lane) = ov;
      if (lane == 0) p.lse[qrow0 + g] = lv;
    }
    __syncwarp();
    __threadfence_block();
    if (lane == 0) {
      sm.ticket[buf] = 0;
      *reinterpret_cast<volatile int*>(&sm.merged[buf]) = (ul >> 1) + 1;
    }
  }
}

template <int G>
cudaError_t launch_g(const ShortParams& p, int sms, int max_ctas, bool after_kernel, cudaStream_t st) {
  // 228 KB of shared memory per SM, 1 KB of it reserved per resident CTA
  static_assert(ShortCfg<G>::kCtasPerSm * (sizeof(ShortSmem<G>) + 1024) <= 228 * 1024, "shared memory per SM");
  const int smem = static_cast<int>(sizeof(ShortSmem<G>));
  static const cudaError_t attr = cudaFuncSetAttribute(reinterpret_cast<const void*>(&short_decode_kernel<G>),
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (attr != cudaSuccess) return attr;
  const int units = p.n_kv_heads * p.n_seq;
  int ctas = ShortCfg<G>::kCtasPerSm * sms;
  if (max_ctas > 0) ctas = min(ctas, max_ctas);
  ctas = max(1, min(ctas, units));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = la;
  cfg.numAttrs = after_kernel ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, short_decode_kernel<G>, p);
}

}  // namespace

cudaError_t launch_short_decode(int G, const ShortParams& p, int sms, int max_ctas, bool after_kernel,
                                cudaStream_t st) {
  if (p.n_seq <= 0 || p.n_kv_heads <= 0) return cudaSuccess;
  switch (G) {
    case 1: return launch_g<1>(p, sms, max_ctas, after_kernel, st);
    case 2: return launch_g<2>(p, sms, max_ctas, after_kernel, st);
    case 4: return launch_g<4>(p, sms, max_ctas, after_kernel, st);
    case 8: return launch_g<8>(p, sms, max_ctas, after_kernel, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ta
