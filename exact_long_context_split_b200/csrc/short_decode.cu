// Decode over many short (sequence, KV head) units: one 4-warp CTA per unit, no shared-memory
// ring.  It serves the suffix part of shared-prefix decode (Bifurcated attention summary,
// briefgpt.xyz, 2403.08845, TL;DR: the per-sample decoded tokens are a second, separate
// product), where hundreds of units of a few hundred tokens each leave the split kernel's
// per-tile pipeline latency-bound.  Every unit is resident at once (a few CTAs per SM), each
// warp streams its quarter of the unit's keys with plain 16-byte loads, and the result folds in
// the prefix pass's chunk statistics before it is written (their exact merge: max and
// logsumexp are associative, Tree Attention article, m.srwj168.com.cn, "The energy view of
// attention").
//
// Per warp, per chunk of 32 keys (online softmax of the "Attention acceleration" concept page,
// compassingai.com, Technical principles 2.1, in base 2, O kept unnormalised):
//   scores:  lane j holds key c0 + j: x_g = (q_g s log2 e) . k for the G query heads of the unit
//   softmax: chunk max per head (warp shuffles); the running max m_g moves only when the chunk's
//            exceeds it by more than 8 (lazy rescale: exact, l and o share the reference)
//   p V:     lane j holds output columns 4 j .. 4 j + 3; key i's weight comes from lane i
// then the 4 warps' (m, l, o) merge in a fixed order in shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "short_decode.h"

namespace ta {
namespace {

constexpr int kD = 128;
constexpr int kWarps = 4;
constexpr float kShortRescale = 8.0f;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

template <int G>
__global__ void __launch_bounds__(kWarps * 32, 4) short_decode_kernel(const __grid_constant__ ShortParams p) {
  __shared__ __align__(16) float qs[G][kD];  // q * scale * log2(e)
  __shared__ float wm[kWarps][G], wl[kWarps][G];
  __shared__ __align__(16) float wo[kWarps][G][kD];
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t S = p.seq_len[b];
  const __nv_bfloat16* K = p.k + p.kv_off[b] + static_cast<int64_t>(h) * S * kD;
  const __nv_bfloat16* V = p.v + p.kv_off[b] + static_cast<int64_t>(h) * S * kD;
  const int64_t qrow0 = static_cast<int64_t>(b) * p.n_q_heads + h * G;  // first output row of the unit

  for (int i = tid; i < G * kD; i += kWarps * 32)
    qs[i / kD][i % kD] = __bfloat162float(p.q[qrow0 * kD + i]) * p.scale_log2;
  __syncthreads();

  const int64_t t0 = warp * S / kWarps, t1 = (warp + 1) * S / kWarps;
  float m[G], lp[G], acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    lp[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = 0.f;
  }
  for (int64_t c0 = t0; c0 < t1; c0 += 32) {
    const int nk = static_cast<int>(min(static_cast<int64_t>(32), t1 - c0));
    const bool valid = lane < nk;
    // scores: the lane's key row in two halves of 128 bytes, each half's 8 loads in flight together
    const uint4* krow = reinterpret_cast<const uint4*>(K + (c0 + lane) * kD);
    float s0[G], s1[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s0[g] = s1[g] = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint4 kr[kD / 16];
#pragma unroll
      for (int e = 0; e < kD / 16; ++e) kr[e] = valid ? __ldg(krow + half * (kD / 16) + e) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int e = 0; e < kD / 16; ++e) {
          const int c = 8 * (half * (kD / 16) + e);  // first column of chunk e
          const float4 qa = *reinterpret_cast<const float4*>(&qs[g][c]);
          const float4 qb = *reinterpret_cast<const float4*>(&qs[g][c + 4]);
          s0[g] = fmaf(qa.x, bf_lo(kr[e].x), s0[g]);
          s1[g] = fmaf(qa.y, bf_hi(kr[e].x), s1[g]);
          s0[g] = fmaf(qa.z, bf_lo(kr[e].y), s0[g]);
          s1[g] = fmaf(qa.w, bf_hi(kr[e].y), s1[g]);
          s0[g] = fmaf(qb.x, bf_lo(kr[e].z), s0[g]);
          s1[g] = fmaf(qb.y, bf_hi(kr[e].z), s1[g]);
          s0[g] = fmaf(qb.z, bf_lo(kr[e].w), s0[g]);
          s1[g] = fmaf(qb.w, bf_hi(kr[e].w), s1[g]);
        }
      }
    }
    float x[G];
#pragma unroll
    for (int g = 0; g < G; ++g) x[g] = valid ? s0[g] + s1[g] : -INFINITY;
    // online softmax (base 2), lazy rescale
    float pg[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float cm = warp_max(x[g]);
      if (cm > m[g] + kShortRescale) {
        const float a = (m[g] == -INFINITY) ? 0.f : ex2(m[g] - cm);
        m[g] = cm;
        lp[g] *= a;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] *= a;
      }
      pg[g] = valid ? ex2(x[g] - m[g]) : 0.f;
      lp[g] += pg[g];
    }
    // p V: lane j owns columns 4 j .. 4 j + 3; V rows loaded 8 at a time
    const uint2* vcol = reinterpret_cast<const uint2*>(V + c0 * kD) + lane;
    for (int j0 = 0; j0 < nk; j0 += 8) {
      uint2 vr[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) vr[u] = (j0 + u < nk) ? __ldg(vcol + (j0 + u) * (kD / 4)) : make_uint2(0, 0);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float v0 = bf_lo(vr[u].x), v1 = bf_hi(vr[u].x), v2 = bf_lo(vr[u].y), v3 = bf_hi(vr[u].y);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float w = __shfl_sync(0xffffffffu, pg[g], j0 + u);  // 0 past the chunk's keys
          acc[g][0] = fmaf(w, v0, acc[g][0]);
          acc[g][1] = fmaf(w, v1, acc[g][1]);
          acc[g][2] = fmaf(w, v2, acc[g][2]);
          acc[g][3] = fmaf(w, v3, acc[g][3]);
        }
      }
    }
  }
  // the warp's statistics
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float l = warp_sum(lp[g]);
    if (lane == 0) {
      wm[warp][g] = m[g];
      wl[warp][g] = l;
    }
    *reinterpret_cast<float4*>(&wo[warp][g][4 * lane]) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  }
  __syncthreads();
  // merge the warps in order, fold in the prefix chunks, write out = o / l and lse.  The row
  // statistics first (one thread per row: the max over warps and chunks, the weights, l), then
  // every thread a float4 of columns with all of its chunk loads independent.
  __shared__ float rM[G], rL[G], rw[G][kWarps];
  __shared__ float cm[G][kShortMaxChunks], cw[G][kShortMaxChunks];  // chunk m, then its weight
  __shared__ float cl[G][kShortMaxChunks];
  const bool fold = p.pre_part != nullptr;
  const int nc = fold ? p.pre_chunks : 0;
  const int64_t cstride = static_cast<int64_t>(p.n_kv_heads) * p.pre_rows * p.pre_stride;
  auto chunk_row = [&](int g) {
    return p.pre_part + (static_cast<int64_t>(h) * p.pre_rows + b * G + g) * p.pre_stride;
  };
  for (int i = tid; i < G * nc; i += kWarps * 32) {  // every chunk's (m, l) of every row at once
    const int g = i / nc, c = i % nc;
    const float* pc = chunk_row(g) + c * cstride;
    cm[g][c] = pc[0];
    cl[g][c] = pc[1];
  }
  __syncthreads();
  if (tid < G) {
    const int g = tid;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w][g]);
    for (int c = 0; c < nc; ++c) M = fmaxf(M, cm[g][c]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float a = (wm[w][g] == -INFINITY) ? 0.f : ex2(wm[w][g] - M);
      rw[g][w] = a;
      L += a * wl[w][g];
    }
    for (int c = 0; c < nc; ++c) {
      const float a = (cm[g][c] == -INFINITY) ? 0.f : ex2(cm[g][c] - M);
      cw[g][c] = a;
      L += a * cl[g][c];
    }
    rM[g] = M;
    rL[g] = L;
  }
  __syncthreads();
  const bool prefix_failed = fold && *reinterpret_cast<const volatile int*>(p.err) != 0;
  for (int i = tid; i < G * (kD / 4); i += kWarps * 32) {
    const int g = i / (kD / 4), d4 = (i % (kD / 4)) * 4;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float a = rw[g][w];
      const float4 o = *reinterpret_cast<const float4*>(&wo[w][g][d4]);
      O = make_float4(O.x + a * o.x, O.y + a * o.y, O.z + a * o.z, O.w + a * o.w);
    }
    if (fold) {
      const float* pre = chunk_row(g) + 4 + d4;
#pragma unroll 6
      for (int c = 0; c < p.pre_chunks; ++c) {
        const float a = cw[g][c];
        const float4 o = *reinterpret_cast<const float4*>(pre + c * cstride);
        O = make_float4(O.x + a * o.x, O.y + a * o.y, O.z + a * o.z, O.w + a * o.w);
      }
    }
    const float L = rL[g];
    float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
    float lv = -INFINITY;
    if (L > 0.f) {
      const float inv = 1.f / L;
      ov = make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
      lv = (rM[g] + log2f(L)) * 0.693147180559945309f;
    }
    if (prefix_failed || L != L) {
      const float nan = __int_as_float(0x7fc00000);
      ov = make_float4(nan, nan, nan, nan);
      lv = nan;
    }
    *reinterpret_cast<float4*>(p.out + (qrow0 + g) * kD + d4) = ov;
    if (d4 == 0) p.lse[qrow0 + g] = lv;
  }
}

}  // namespace

cudaError_t launch_short_decode(int G, int n_kv_heads, int batch, const ShortParams& p, cudaStream_t st) {
  const dim3 grid(n_kv_heads, batch);
  switch (G) {
    case 1: short_decode_kernel<1><<<grid, kWarps * 32, 0, st>>>(p); break;
    case 2: short_decode_kernel<2><<<grid, kWarps * 32, 0, st>>>(p); break;
    case 4: short_decode_kernel<4><<<grid, kWarps * 32, 0, st>>>(p); break;
    case 8: short_decode_kernel<8><<<grid, kWarps * 32, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace ta
