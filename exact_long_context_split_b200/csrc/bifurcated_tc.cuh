// Bifurcated decode, shared-prefix part, on the 5th-generation tensor cores.
//
// Bifurcated attention summary (briefgpt.xyz, 2403.08845, TL;DR): when many samples
// decode from one prefilled context, the attention over that shared context is one
// dense product of all the samples' queries with the context keys, kept exact; the
// samples' own decoded tokens are a second, separate product.  Per KV head h the
// queries of every sample n and every query head g of the group form the rows
// r = n * G + g of one matrix Q_h, so the context part is
//     S = Q_h K_h^T,   online softmax over the context,   O = P V_h
// ("Attention acceleration" concept page, compassingai.com, Technical principles 2.1:
// tiles of keys, running max m and sum l, output rescaled when m grows).
//
// Each CTA writes per row the statistics (m in log2 units, l, unnormalised o) of its
// chunk; the suffix pass (split kernel) folds them into each row as it writes the result.
//
// One CTA owns up to 256 rows (two M tiles of 128) and a contiguous chunk of 128-key
// tiles of the context; both M tiles consume every K/V tile it loads.
// Roles (12 warps):  warp 0 lane 0: TMA producer (K(t) then V(t), each refilling a stage once
// its products freed it);  warp 1: TMEM allocation, lane 0 issues tcgen05.mma in a fixed
// order.  Both block on one barrier at a time (suspending try_wait) rather than polling every
// condition: spinning would take issue slots from the two softmax warps that share each of
// their SM sub-partitions (a fixed order measured 8% faster on the shared-prefix step);
// warps 2-3: convert each V tile from bf16 to fp16 in place (P is fp16 for the P V
// product: bf16 P is too coarse, and one MMA needs A and B of the same type);  warps 4-7
// and 8-11: softmax of M tile 0 and 1, thread t owns row t = TMEM lane t.
// TMEM columns: S of tile w at 128 w (fp32, 128 x 128); P (fp16, two per column)
// overwrites its first 64 columns and is the A operand of P V; O of tile w at 256 + 128 w.
// Per M tile the MMA thread alternates S(t) = Q K(t)^T and O += P(t) V(t); the tensor pipe
// runs them in issue order, so S(t + 1) landing also means P(t) V(t) is complete.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "bifurcated_tc.h"
#include "ptx.cuh"

namespace ta {

constexpr int kBifKStages = 3;      // K ring depth (K frees a stage after S = Q K^T)
constexpr int kBifVStages = 2;      // V ring depth (V frees a stage after O += P V)
constexpr int kBifTmemCols = 512;   // S: 2 tiles x 128 columns; O: 2 tiles x 128 columns
constexpr float kBifRescale = 8.0f;  // lazy rescaling threshold (log2 units)
// The two softmax warpgroups may take turns on the exponentials (a per-tile handoff); measured
// without the handoff on one B200: the shared-prefix pass 86.7 against 88.8 us, context encoding
// 6,441 against 6,592 us (32K), several query tokens 172.8 against 177.0 us.
constexpr bool kBifPingPong = false;


struct BifSmem {
  alignas(1024) uint8_t q[kBifMT][2][kBifRows * 128];        // bf16 Q tiles, two 64-column blocks each, SW128
  alignas(1024) uint8_t k[kBifKStages][2][kBifKeys * 128];   // bf16 K tiles, two 64-column blocks
  alignas(1024) uint8_t v[kBifVStages][2][kBifKeys * 128];   // V tiles (bf16 -> fp16 in place), MN-major
  uint64_t k_full[kBifKStages], k_empty[kBifKStages];
  uint64_t v_full[kBifVStages], v_conv[kBifVStages], v_empty[kBifVStages];
  uint64_t s_full[kBifMT], p_full[kBifMT], o_done[kBifMT];
  uint64_t turn[kBifMT];  // turn[w] completes a phase when the other M tile's exponentials are done
  uint64_t q_ready, mma_idle;
  uint32_t tmem_base;
  int abort;
};


// ---------------------------------------------------------------------------------------------
// PTX wrappers (tcgen05, TMA tensor loads, proxy fences)
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] x B[smem desc]; `accumulate` false overwrites D.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           bool accumulate) {
  const uint32_t acc = accumulate ? 1u : 0u;
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem desc]; A is K-major in TMEM (row = lane, two 16-bit
// elements per 32-bit column).
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              bool accumulate) {
  const uint32_t acc = accumulate ? 1u : 0u;
  const uint32_t z = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc), "r"(z), "r"(z), "r"(z), "r"(z)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version 1.
// lbo/sbo in bytes: for K-major operands sbo is the stride between 8-row groups (lbo unused);
// for MN-major operands lbo is the stride between 64-element blocks of the MN dimension and
// sbo the stride between 8-row groups of the K dimension.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3fff);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3fff) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor of tcgen05.mma kind::f16 with an f32 accumulator.
// a_bf16/b_bf16: operand type (bf16 or fp16); b_mn_major: B stored MN-major.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N, bool a_bf16, bool b_bf16, bool b_mn_major) {
  return (1u << 4) | ((a_bf16 ? 1u : 0u) << 7) | ((b_bf16 ? 1u : 0u) << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128-byte-swizzled block of rows.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// 3-input max / min (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// tcgen05.wait::ld that also hands the loaded registers through, so no use of them can be
// scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld_regs(float (&v)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]), "+f"(v[8]),
        "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]),
        "+f"(v[17]), "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]), "+f"(v[24]),
        "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]), "+f"(v[30]), "+f"(v[31])
      :
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Scaled max of a full tile's 128 scores (the raw extreme times the scale: for a negative
// scale the raw minimum), two 32-column loads at a time, four independent chains.
__device__ __forceinline__ float bif_tile_max(uint32_t s_col, float sc) {
  float a[32], b[32];
  float e[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    tmem_ld32(s_col + 64 * h, a);
    tmem_ld32(s_col + 64 * h + 32, b);
    tmem_wait_ld_regs(a);
    tmem_wait_ld_regs(b);
    if (h == 0) {
#pragma unroll
      for (int k = 0; k < 4; ++k) e[k] = a[k];
    }
    if (sc >= 0.f) {
#pragma unroll
      for (int c = (h == 0 ? 4 : 0); c < 32; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) e[k] = fmax3(e[k], a[c + k], c + k + 4 < 32 ? a[c + k + 4] : a[c + k]);
      }
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) e[k] = fmax3(e[k], b[c + k], b[c + k + 4]);
      }
    } else {
#pragma unroll
      for (int c = (h == 0 ? 4 : 0); c < 32; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) e[k] = fmin3(e[k], a[c + k], c + k + 4 < 32 ? a[c + k + 4] : a[c + k]);
      }
#pragma unroll
      for (int c = 0; c < 32; c += 8) {
#pragma unroll
        for (int k = 0; k < 4; ++k) e[k] = fmin3(e[k], b[c + k], b[c + k + 4]);
      }
    }
  }
  const float x = sc >= 0.f ? fmax3(e[0], e[1], fmaxf(e[2], e[3])) : fmin3(e[0], e[1], fminf(e[2], e[3]));
  return x * sc;
}

// The last, partial tile of the context: keys at or past `nvalid` do not exist.
__device__ __forceinline__ float bif_tile_max_partial(uint32_t s_col, float sc, int nvalid) {
  float tmax = -INFINITY;
#pragma unroll 1
  for (int q = 0; q < kBifKeys / 32; ++q) {
    float a[32];
    tmem_ld32(s_col + 32 * q, a);
    tmem_wait_ld_regs(a);
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (32 * q + c < nvalid) tmax = fmaxf(tmax, a[c] * sc);
  }
  return tmax;
}

// 32 scores -> 16 fp16 pairs of p = 2^(x s - mn) at P columns [col, col + 16); adds p to acc.
__device__ __forceinline__ void bif_exp_chunk(const float (&x)[32], uint32_t col, float2 s2, float2 nm,
                                              float2 (&acc)[4]) {
  uint32_t h[16];
#pragma unroll
  for (int c2 = 0; c2 < 16; ++c2) {
    const float2 y = __ffma2_rn(make_float2(x[2 * c2], x[2 * c2 + 1]), s2, nm);
    const float2 pp = make_float2(ex2(y.x), ex2(y.y));
    acc[c2 & 3] = __fadd2_rn(acc[c2 & 3], pp);
    const __half2 hv = __floats2half2_rn(pp.x, pp.y);
    h[c2] = *reinterpret_cast<const uint32_t*>(&hv);
  }
  tmem_st16u(col, h);
}

// Pass 2 over a full tile, 32 scores at a time.  P chunk q goes to columns [16 q, 16 q + 16),
// below every score column still to be read.  (Loading the next 32 scores while the current
// ones are exponentiated held two 32-column buffers and spilled registers to local memory on
// this path, where each spill is an L2 round trip beside 224 KB of shared memory; the
// one-buffer loop does the same operations in the same order without spills, and measured
// 0.5-1% faster on every mode.)
__device__ __forceinline__ float bif_tile_exp(uint32_t s_col, float sc, float mn) {
  const float2 s2 = make_float2(sc, sc), nm = make_float2(-mn, -mn);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float a[32];
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    tmem_ld32(s_col + 32 * q, a);
    tmem_wait_ld_regs(a);
    bif_exp_chunk(a, s_col + 16 * q, s2, nm, acc);
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  const float2 a4 = __fadd2_rn(a01, a23);
  return a4.x + a4.y;
}

__device__ __forceinline__ float bif_tile_exp_partial(uint32_t s_col, float sc, float mn, int nvalid) {
  float rs = 0.f;
#pragma unroll 1
  for (int q = 0; q < kBifKeys / 32; ++q) {
    float a[32];
    tmem_ld32(s_col + 32 * q, a);
    tmem_wait_ld_regs(a);
    uint32_t h[16];
#pragma unroll
    for (int c2 = 0; c2 < 16; ++c2) {
      const int c = 32 * q + 2 * c2;
      const float p0 = (c < nvalid) ? ex2(a[2 * c2] * sc - mn) : 0.f;
      const float p1 = (c + 1 < nvalid) ? ex2(a[2 * c2 + 1] * sc - mn) : 0.f;
      rs += p0 + p1;
      const __half2 hv = __floats2half2_rn(p0, p1);
      h[c2] = *reinterpret_cast<const uint32_t*>(&hv);
    }
    tmem_st16u(s_col + 16 * q, h);
  }
  return rs;
}

// Bounded wait shared by every role: gives up after limit_ns or once the CTA aborted.
__device__ __forceinline__ bool bif_wait(uint64_t* bar, uint32_t parity, const BifParams& p, volatile int* abort) {
  if (*abort) return false;
  if (wait_phase(bar, parity, p.wait_limit_ns, abort)) return true;
  if (!*abort) atomicCAS(p.err, 0, kErrBifWait);
  *abort = 1;
  return false;
}


// ---------------------------------------------------------------------------------------------
// The prefix kernel
// ---------------------------------------------------------------------------------------------

// PAGED: mode 1 over a paged cache (a separate instance: the contiguous kernel carries none of
// the paged producer's code).
template <bool PAGED>
__global__ void __launch_bounds__(kBifThreads, 1)
    bif_prefix_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ BifParams p) {
  extern __shared__ __align__(16) uint8_t bif_smem_raw[];
  // 128-byte swizzling needs 1024-byte aligned tiles in the shared window.
  const uint32_t raw = smem_addr(bif_smem_raw);
  BifSmem& sm = *reinterpret_cast<BifSmem*>(bif_smem_raw + (((raw + 1023u) & ~1023u) - raw));

  // A kernel launched after this one with programmatic dependent launch (the short-unit suffix
  // pass) may start on the SMs this grid leaves free; it waits for this grid's completion before
  // it reads anything this kernel writes.
  asm volatile("griddepcontrol.launch_dependents;");
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // The CTA's unit: its rows, its keys (a range of tensor-map rows) and its chunk of them.
  const bool multi = p.mode == 1;
  const bool anchor = p.mode == 2;
  const int chunk = multi ? blockIdx.x : (anchor ? 0 : blockIdx.y);
  const int h = multi || anchor ? blockIdx.y : blockIdx.z;
  const int b = multi ? blockIdx.z : 0;
  const int row0 = multi || anchor ? 0 : blockIdx.x * kBifMT * kBifRows;  // first row of this CTA in the unit
  // Mode 0: M tile w holds rows row0 + 128 w + lane and reads every key tile.  Modes 1 and 2:
  // both slots hold the unit's rows; slot w reads key tiles w, w + 2, ... ("split" slots).
  const int n_mt = multi || anchor ? 1 : min(kBifMT, (p.rows_per_head - row0 + kBifRows - 1) / kBifRows);
  const bool split = multi || anchor;
  const int n_slots = split ? kBifMT : n_mt;
  // Mode 2: query tile qt (launched last tile first: the later blocks see the most keys) holds
  // positions p0 .. p0 + n_pos - 1 of context block blk; its keys are the virtual sequence
  // [anchor block ; own block up to its last position] (no anchor for the first block).
  const int64_t qt = anchor ? static_cast<int64_t>(gridDim.x) - 1 - blockIdx.x : 0;
  const int64_t p0 = qt * p.n_pos;
  const int n_tok = anchor ? static_cast<int>(min(static_cast<int64_t>(p.n_pos), p.ctx_len - p0))
                           : (multi ? p.n_queries : 1);  // query tokens of the unit
  const int64_t blk = anchor ? p0 / p.block_size : 0;
  const int64_t anchor_len = blk > 0 ? p.block_size : 0;  // keys of the anchor segment
  const int64_t own0 = blk * p.block_size;                 // first key of the own segment
  const int64_t kv_len = multi ? p.kv_len[b] : (anchor ? anchor_len + (p0 + n_tok - own0) : p.prefix_len);
  const int64_t kv_row0 = multi ? p.kv_row0[b] + h * kv_len
                                : static_cast<int64_t>(h) * (anchor ? p.ctx_len : p.prefix_len);
  const int64_t q_tok0 = multi ? static_cast<int64_t>(b) * p.n_queries : p0;  // q row of the unit's first token
  const int64_t n_tiles = (kv_len + kBifKeys - 1) / kBifKeys;
  const int64_t j0 = chunk * n_tiles / p.n_chunks;
  const int n_t = static_cast<int>((chunk + 1) * n_tiles / p.n_chunks - j0);
  // Tensor-map row of key tile t of the CTA's chunk (mode 2: the anchor segment, then the own
  // one; block_size is a multiple of the tile, so no tile spans both).
  auto tile_row = [&](int t) -> int {
    const int64_t v = (j0 + t) * kBifKeys;
    if (!anchor || v < anchor_len) return static_cast<int>(kv_row0 + v);
    return static_cast<int>(kv_row0 + own0 + (v - anchor_len));
  };
  // Test hook: CTA (0, 0, 0) never loads this K tile, so the products that need it wait in vain.
  const int skip_tile = (blockIdx.x | blockIdx.y | blockIdx.z) == 0 ? p.debug_skip_tile1 - 1 : -1;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kBifKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], split ? 1 : n_mt);  // one commit per S = Q K^T that reads it
    }
#pragma unroll
    for (int s = 0; s < kBifVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_conv[s], 64);
      mbar_init(&sm.v_empty[s], split ? 1 : n_mt);  // one commit per O += P V that reads it
    }
#pragma unroll
    for (int w = 0; w < kBifMT; ++w) {
      mbar_init(&sm.s_full[w], 1);
      mbar_init(&sm.p_full[w], kBifRows);
      mbar_init(&sm.o_done[w], 1);
      mbar_init(&sm.turn[w], kBifRows);
    }
    mbar_init(&sm.q_ready, kBifMT * kBifRows);
    mbar_init(&sm.mma_idle, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm.tmem_base)),
                 "r"(kBifTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------
    // K and V tiles in order; a K stage refills once every S = Q K^T that reads it is done, a
    // V stage once every P V that reads it is done.  Contiguous: lane 0 alone.  Paged: the
    // whole warp, lane k issuing the k-th page segment's boxes.
    if (PAGED || lane == 0) {
      uint64_t pol;
      if (anchor)  // every key tile is read by many query tiles: keep it in L2
        asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
      else
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
      int fk[kBifKStages] = {}, fv[kBifVStages] = {};  // copies issued per stage
      if constexpr (!PAGED) {
        auto issue = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* full, int t) {
          const int y = tile_row(t);
          mbar_arrive_expect_tx(full, 2 * kBifKeys * 128);
          tma_load_2d(dst, map, 0, y, full, pol);
          tma_load_2d(dst + kBifKeys * 128, map, 64, y, full, pol);
        };
        // K(t) once every product that read K(t - 3) is done, then V(t) once P V(t - 2) is.
        for (int t = 0; t < n_t && !*abort; ++t) {
          if (t >= kBifKStages && !bif_wait(&sm.k_empty[t % kBifKStages], ((t / kBifKStages) - 1) & 1, p, abort))
            break;
          if (t != skip_tile) {
            issue(&kmap, sm.k[t % kBifKStages][0], &sm.k_full[t % kBifKStages], t);
            ++fk[t % kBifKStages];
          }
          if (t >= kBifVStages && !bif_wait(&sm.v_empty[t % kBifVStages], ((t / kBifVStages) - 1) & 1, p, abort))
            break;
          issue(&vmap, sm.v[t % kBifVStages][0], &sm.v_full[t % kBifVStages], t);
          ++fv[t % kBifVStages];
        }
      } else {
        // A tile is n_sub boxes of bs rows: one box of 128 rows of a contiguous cache, or one per
        // page segment of a paged one (the 128-byte swizzle repeats every 8 rows, so boxes of 16
        // or more rows at their row offsets build the same tile layout as one 128-row box).
        const int bs = min(1 << p.log2_page, kBifKeys);
        const int n_sub = kBifKeys / bs;  // boxes per half-tile, at most 8 (pages of 16+ tokens)
        const int64_t last_blk = (kv_len - 1) >> p.log2_page;
        int32_t pg = 0;  // this lane's block-table entry of the next tile, loaded ahead
        int y = 0;       // this lane's box row of the current tile
        // Lane k loads tile t's k-th entry; the value is used only in resolve(t), after the stage
        // wait, so the load's latency overlaps it.  Boxes past the sequence's end read its last
        // block (their keys are masked and their V rows zeroed).
        auto fetch = [&](int t) {
          if (lane < n_sub) {
            const int64_t blk = ((j0 + t) * kBifKeys + static_cast<int64_t>(lane) * bs) >> p.log2_page;
            pg = __ldg(p.block_table + b * p.bt_stride + min(blk, last_blk));
          }
        };
        // Box rows of tile t; false (for every lane) if any entry is outside the pool.
        auto resolve = [&](int t) -> bool {
          bool good = true;
          if (lane < n_sub) {
            const int64_t tok = (j0 + t) * kBifKeys + static_cast<int64_t>(lane) * bs;
            const int64_t blk = tok >> p.log2_page;
            const int64_t page = pg;
            good = page >= 0 && page < p.num_pages;
            const int64_t off = blk > last_blk ? 0 : (tok & ((int64_t(1) << p.log2_page) - 1));
            y = static_cast<int>(((page * p.n_kv_heads + h) << p.log2_page) + off);
          }
          return __all_sync(0xffffffffu, good);
        };
        auto issue = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* full) {
          if (lane == 0) mbar_arrive_expect_tx(full, 2 * kBifKeys * 128);
          __syncwarp();
          if (lane < n_sub) {
            tma_load_2d(dst + lane * bs * 128, map, 0, y, full, pol);
            tma_load_2d(dst + kBifKeys * 128 + lane * bs * 128, map, 64, y, full, pol);
          }
        };
        auto stage_wait = [&](uint64_t* bar, uint32_t parity) -> bool {  // lane 0 waits, all learn
          bool ok = true;
          if (lane == 0) ok = bif_wait(bar, parity, p, abort);
          return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        };
        if (n_t > 0) fetch(0);
        // K(t) once every product that read K(t - 3) is done, then V(t) once P V(t - 2) is.
        for (int t = 0; t < n_t; ++t) {
          if (__shfl_sync(0xffffffffu, *abort ? 1 : 0, 0) != 0) break;
          if (t >= kBifKStages && !stage_wait(&sm.k_empty[t % kBifKStages], ((t / kBifKStages) - 1) & 1)) break;
          if (!resolve(t)) {  // checked before anything is expected on the stage's barrier
            if (lane == 0) {
              atomicCAS(p.err, 0, kErrBifBadPage);
              *abort = 1;
            }
            break;
          }
          if (t + 1 < n_t) fetch(t + 1);
          issue(&kmap, sm.k[t % kBifKStages][0], &sm.k_full[t % kBifKStages]);
          ++fk[t % kBifKStages];
          if (t >= kBifVStages && !stage_wait(&sm.v_empty[t % kBifVStages], ((t / kBifVStages) - 1) & 1)) break;
          issue(&vmap, sm.v[t % kBifVStages][0], &sm.v_full[t % kBifVStages]);
          ++fv[t % kBifVStages];
        }
      }
      // Every issued copy lands before the CTA moves on: stage s completed one phase per copy
      // issued to it, so the last of them has parity (count - 1) & 1.
      if (lane == 0) {
        for (int s = 0; s < kBifKStages; ++s)
          if (fk[s] > 0 && !wait_phase(&sm.k_full[s], (fk[s] - 1) & 1, p.wait_limit_ns, nullptr))
            atomicCAS(p.err, 0, kErrBifWait);
        for (int s = 0; s < kBifVStages; ++s)
          if (fv[s] > 0 && !wait_phase(&sm.v_full[s], (fv[s] - 1) & 1, p.wait_limit_ns, nullptr))
            atomicCAS(p.err, 0, kErrBifWait);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------- MMA issuer ---------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = f16_idesc(kBifRows, kBifKeys, true, true, false);
      constexpr uint32_t idesc_pv = f16_idesc(kBifRows, kBifD, false, false, true);
      bool ok = bif_wait(&sm.q_ready, 0, p, abort);
      tc_fence_after();
      // Per M tile w the stream is S(0), PV(0), S(1), PV(1), ...: S(t + 1) overwrites the
      // TMEM columns where P(t) was read, so it follows P(t) V(t) in issue order.
      int nw[kBifMT];  // key tiles of each slot; a slot's local tile t is the CTA's tile t or 2 t + w
      for (int w = 0; w < kBifMT; ++w) nw[w] = w >= n_slots ? 0 : (split ? (n_t - w + 1) / 2 : n_t);
      {
        // Slot w's S(i) = Q K(i)^T and O += P(i) V(i), i the slot's local key tile.
        auto qk = [&](int w, int i) -> bool {
          const int t = split ? 2 * i + w : i, s = t % kBifKStages;
          if (!bif_wait(&sm.k_full[s], (t / kBifKStages) & 1, p, abort)) return false;
          tc_fence_after();
          const uint32_t q_base = smem_addr(sm.q[split ? 0 : w]);
          const uint32_t k_base = smem_addr(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < kBifD / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 16-element K step inside a 128-byte row
            const uint64_t a = sw128_desc(q_base + (kk >> 2) * (kBifRows * 128) + off, 16, 1024);
            const uint64_t bd = sw128_desc(k_base + (kk >> 2) * (kBifKeys * 128) + off, 16, 1024);
            tc_mma_f16(tmem + w * 128, a, bd, idesc_qk, kk > 0);
          }
          tc_commit(&sm.s_full[w]);
          tc_commit(&sm.k_empty[s]);
          return true;
        };
        auto pv = [&](int w, int i) -> bool {
          const int t = split ? 2 * i + w : i, s = t % kBifVStages;
          if (!bif_wait(&sm.v_conv[s], (t / kBifVStages) & 1, p, abort)) return false;
          if (!bif_wait(&sm.p_full[w], i & 1, p, abort)) return false;
          tc_fence_after();
          const uint32_t v_base = smem_addr(sm.v[s]);
#pragma unroll
          for (int kk = 0; kk < kBifKeys / 16; ++kk) {
            const uint64_t bd = sw128_desc(v_base + kk * 16 * 128, kBifKeys * 128, 1024);
            tc_mma_f16_ts(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, bd, idesc_pv, i > 0 || kk > 0);
          }
          tc_commit(&sm.v_empty[s]);
          if (i == nw[w] - 1) tc_commit(&sm.o_done[w]);
          return true;
        };
        // S of each slot's first tile, then per tile i and slot w, P V(i) and S(i + 1): the
        // slots start a tile's softmax in the order slot 0, slot 1, and about as long each.
        for (int w = 0; ok && w < n_slots; ++w)
          if (nw[w] > 0) ok = qk(w, 0);
        const int n_rounds = max(nw[0], nw[1]);
        for (int i = 0; ok && i < n_rounds; ++i) {
          for (int w = 0; ok && w < n_slots; ++w) {
            if (i < nw[w]) ok = pv(w, i);
            if (ok && i + 1 < nw[w]) ok = qk(w, i + 1);
          }
        }
      }
      // Every issued MMA completes before the tensor memory is released.
      tc_commit(&sm.mma_idle);
      if (!wait_phase(&sm.mma_idle, 0, p.wait_limit_ns, nullptr)) atomicCAS(p.err, 0, kErrBifWait);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------- V converters -------------------------------
    const int ct = tid - 64;
    for (int i = 0; i < n_t; ++i) {
      const int s = i % kBifVStages;
      if (!bif_wait(&sm.v_full[s], (i / kBifVStages) & 1, p, abort)) break;
      uint4* v4 = reinterpret_cast<uint4*>(sm.v[s]);
      // Rows past the unit's keys hold whatever follows it (another head, a free page): their
      // scores are masked, but 0 * NaN is NaN in P V, so they are zeroed.
      const int64_t valid = kv_len - (j0 + i) * static_cast<int64_t>(kBifKeys);
      if (valid < kBifKeys) {
        for (int c = ct; c < 2 * kBifKeys * 128 / 16; c += 64)
          if (((c & 1023) >> 3) >= valid) v4[c] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll 4
      for (int c = ct; c < 2 * kBifKeys * 128 / 16; c += 64) {
        uint4 w = v4[c];
        uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 hv =
              __floats2half2_rn(__uint_as_float(ws[e] << 16), __uint_as_float(ws[e] & 0xffff0000u));
          ws[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        v4[c] = make_uint4(ws[0], ws[1], ws[2], ws[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&sm.v_conv[s]);
    }
  } else {
    // ------------------------------- softmax ------------------------------------
    const int w = (warp - 4) >> 2;                    // M tile of this warpgroup
    const int r = tid - 128 - w * kBifRows;           // row of the M tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + w * 128;
    const uint32_t o_col = tmem + lane_base + 256 + w * 128;
    const int G = p.n_q_heads / p.n_kv_heads;
    const int row = split ? r : row0 + w * kBifRows + r;  // row of the unit's query matrix
    const bool valid_row = row < (anchor ? n_tok * G : p.rows_per_head);
    // Keys at the end of the unit this row may not see (modes 1 and 2: query token j of n is
    // n - 1 - j positions before the last one).
    const int lag = (split && valid_row) ? n_tok - 1 - row / G : 0;
    if (!split || w == 0) {
      const int n = row / G, g = row % G;
      const uint4* src = reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) +
          (static_cast<int64_t>(q_tok0 + n) * p.n_q_heads + h * G + g) * kBifD);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = valid_row ? src[c] : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sm.q[w][c >> 3] + sw128_offset(r, c & 7)) = v;
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&sm.q_ready);
    // A warp none of whose rows is real (few rows per unit, a partial last tile) skips the
    // scores' max and exponentials and the rescaling: its Q rows are zero, so its S rows, and
    // the P rows read over them, are zero.  It still takes every wait and arrival in order.
    const bool active = __any_sync(0xffffffffu, valid_row);
    const float sc = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = w < n_slots;
    const int n_w = w >= n_slots ? 0 : (split ? (n_t - w + 1) / 2 : n_t);
    for (int i = 0; ok && i < n_w; ++i) {
      // S(i) landed; with it, P(i - 1) V(i - 1) is complete (same issuing thread, in order).
      ok = bif_wait(&sm.s_full[w], i & 1, p, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int tg = split ? 2 * i + w : i;  // the CTA's key tile
      const int64_t nvalid64 = kv_len - lag - (j0 + tg) * kBifKeys;
      const int nvalid = static_cast<int>(max(static_cast<int64_t>(-1), min(nvalid64, static_cast<int64_t>(kBifKeys))));
      // tcgen05.ld is warp-collective: a warp takes the masked path if any of its rows needs it.
      const bool full = __all_sync(0xffffffffu, nvalid >= kBifKeys);
      // Pass 1: the tile's scaled row max, streamed from TMEM.
      const float tmax = !active ? -INFINITY : (full ? bif_tile_max(s_col, sc) : bif_tile_max_partial(s_col, sc, nvalid));
      const bool need = tmax > m + kBifRescale;
      const float mn = need ? tmax : m;
      // Ping-pong: M tile 1's exponentials of key tile i follow M tile 0's, and M tile 0's of
      // tile i + 1 follow M tile 1's of tile i, so one warpgroup's exponentials overlap the
      // other M tile's products on the tensor pipe.
      const bool pingpong = kBifPingPong && n_slots == kBifMT;
      if (pingpong && (w == 1 || i >= 1)) {
        ok = bif_wait(&sm.turn[w], (w == 1 ? i : i - 1) & 1, p, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      // Pass 2: p = 2^(x s - m), summed in fp32, written back as fp16 pairs over the first 64
      // columns of S (P overwrites only columns whose scores were already read).
      const float rs = !active ? 0.f : (full ? bif_tile_exp(s_col, sc, mn) : bif_tile_exp_partial(s_col, sc, mn, nvalid));
      if (pingpong) mbar_arrive(&sm.turn[1 - w]);
      const float alpha = (need && m != -INFINITY) ? ex2(m - mn) : 1.f;
      // O holds tiles 0..i-1 and P(i - 1) V(i - 1) is complete: rescale it when m grew.
      if (active && __any_sync(0xffffffffu, need && i >= 1)) {
#pragma unroll
        for (int q4 = 0; q4 < kBifD / 32; ++q4) {
          float o[32];
          tmem_ld32(o_col + q4 * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] *= alpha;
          tmem_st32(o_col + q4 * 32, o);
        }
      }
      tmem_wait_st();
      l = l * alpha + rs;
      m = mn;
      tc_fence_before();
      mbar_arrive(&sm.p_full[w]);
    }
    if (anchor) {
      // Mode 2: both slots hold the same rows over alternate key tiles.  Slot 1 publishes its
      // (m, l) in shared memory (the second Q buffer, unused with split slots); slot 0 merges
      // them with its own, reads both O accumulators from TMEM and writes the final row.
      const int n1 = n_t / 2;  // key tiles of slot 1 (slot 0 has (n_t + 1) / 2 >= 1)
      if (n_w > 0 && ok) {
        ok = bif_wait(&sm.o_done[w], 0, p, abort);
        ok = __all_sync(0xffffffffu, ok);
      }
      float* st = reinterpret_cast<float*>(sm.q[1][0]);
      if (w == 1) {
        st[r] = n1 > 0 ? m : -INFINITY;
        st[kBifRows + r] = n1 > 0 ? l : 0.f;
        st[2 * kBifRows + r] = ok ? 0.f : 1.f;
        tc_fence_before();
      }
      named_barrier(1, 2 * kBifRows);
      if (w == 0) {
        tc_fence_after();
        const float m1 = st[r], l1 = st[kBifRows + r];
        const bool bad = !ok || st[2 * kBifRows + r] != 0.f;
        const float M = fmaxf(m, m1);
        const float a0 = (m == -INFINITY) ? 0.f : ex2(m - M);
        const float a1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - M);
        const float L = l * a0 + l1 * a1;
        const float inv = L > 0.f ? 1.f / L : 0.f;
        const float c0 = a0 * inv, c1 = a1 * inv;
        const float nan = __int_as_float(0x7fc00000);
        const int64_t orow = (q_tok0 + row / G) * p.n_q_heads + h * G + row % G;
        float* dst = p.out + orow * kBifD;
#pragma unroll 1
        for (int q4 = 0; q4 < kBifD / 32; ++q4) {
          float o[32], o1[32];
          tmem_ld32(o_col + q4 * 32, o);  // slot 0 always has a tile (every query sees itself)
          if (n1 > 0) tmem_ld32(o_col + 128 + q4 * 32, o1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = bad ? nan : (n1 > 0 ? o[c] * c0 + o1[c] * c1 : o[c] * c0);
          if (valid_row) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + q4 * 32 + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
          }
        }
        if (valid_row) p.lse[orow] = bad ? nan : (L > 0.f ? (M + log2f(L)) * 0.693147180559945309f : -INFINITY);
      }
    } else if (w < n_slots) {
      // The chunk's statistics of this row.
      // Mode 0: [chunk][KV head][row]; mode 1: [sequence, KV head][chunk][slot][row].
      const int64_t prow =
          multi ? ((static_cast<int64_t>(b) * p.n_kv_heads + h) * p.n_chunks + chunk) * kBifMT + w
                : static_cast<int64_t>(chunk) * p.n_kv_heads + h;
      float* dst = p.part + (prow * p.rows_per_head + row) * kBifPartRow;
      if (n_w > 0 && ok) {
        ok = bif_wait(&sm.o_done[w], 0, p, abort);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (n_w > 0 && ok) {
        tc_fence_after();
#pragma unroll
        for (int q4 = 0; q4 < kBifD / 32; ++q4) {
          float o[32];
          tmem_ld32(o_col + q4 * 32, o);
          tmem_wait_ld();
          if (valid_row) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + 4 + q4 * 32 + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
          }
        }
        if (valid_row) {
          dst[0] = m;
          dst[1] = l;
        }
      } else if (valid_row) {
        // Empty chunk, or an aborted one (the error word is set and the merge writes NaN).
        dst[0] = -INFINITY;
        dst[1] = 0.f;
        for (int c = 0; c < kBifD; ++c) dst[4 + c] = 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kBifTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------------------------------------
// Merge: the prefix chunks' statistics with the suffix result, per (sample, query head)
// ---------------------------------------------------------------------------------------------

// Mode 1: a unit's 2 * n_chunks partials, merged online per output row (b, j, hq); one thread
// per 4 columns.
__global__ void __launch_bounds__(128) merge_chunks_kernel(const float* __restrict__ part, int n_chunks,
                                                           int n_kv_heads, int rows_per_head, int n_queries,
                                                           float* __restrict__ out, float* __restrict__ lse,
                                                           int batch, int n_q_heads, const int* __restrict__ err) {
  constexpr int Q = kBifD / 4;
  // The partials are those of the kernel launched before this one: wait for its completion
  // (immediate when this launch was not a programmatic dependent).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(batch) * n_queries * n_q_heads * Q;
  if (i >= total) return;
  const int d4 = static_cast<int>(i % Q) * 4;
  const int64_t rq = i / Q;  // (b * n + j) * Hq + hq
  const int hq = static_cast<int>(rq % n_q_heads);
  const int64_t bj = rq / n_q_heads;
  const int j = static_cast<int>(bj % n_queries), b = static_cast<int>(bj / n_queries);
  const int G = n_q_heads / n_kv_heads;
  const int h = hq / G, row = j * G + hq % G;
  const int n_parts = n_chunks * kBifMT;
  const float* base = part + ((static_cast<int64_t>(b) * n_kv_heads + h) * n_parts * rows_per_head + row) * kBifPartRow;
  const int64_t stride = static_cast<int64_t>(rows_per_head) * kBifPartRow;
  float M = -INFINITY, L = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int c = 0; c < n_parts; ++c) {
    const float* pc = base + c * stride;
    const float2 ml = *reinterpret_cast<const float2*>(pc);
    const float4 o = *reinterpret_cast<const float4*>(pc + 4 + d4);
    // No branch: a chunk or slot without keys for this row (m = -inf) gets weight 0, so the
    // loads of the whole unrolled group issue together.
    const float Mn = fmaxf(M, ml.x);
    const float a = (M == -INFINITY) ? 0.f : ex2(M - Mn);
    const float bw = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - Mn);
    L = L * a + ml.y * bw;
    O = make_float4(O.x * a + o.x * bw, O.y * a + o.y * bw, O.z * a + o.z * bw, O.w * a + o.w * bw);
    M = Mn;
  }
  float4 ov = make_float4(0.f, 0.f, 0.f, 0.f);
  float lv = -INFINITY;
  if (L > 0.f) {
    ov = make_float4(O.x / L, O.y / L, O.z / L, O.w / L);
    lv = (M + log2f(L)) * 0.693147180559945309f;
  }
  if (*reinterpret_cast<const volatile int*>(err) != 0) {
    const float nan = __int_as_float(0x7fc00000);
    ov = make_float4(nan, nan, nan, nan);
    lv = nan;
  }
  *reinterpret_cast<float4*>(out + rq * kBifD + d4) = ov;
  if (d4 == 0) lse[rq] = lv;
}

}  // namespace ta
