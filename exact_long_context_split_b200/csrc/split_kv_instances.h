// Host-side handle of the compiled split-KV kernel instances.  Each (element type, tile
// configuration, head_dim, contiguous or paged cache) is compiled in a translation unit of
// its own (split_kv_[paged_]<type>_<tiles>_d<D>.cu) so that the instances build in parallel.
#pragma once
#include <cuda_bf16.h>

#include <cstddef>

#include "split_kv.cuh"

namespace ta {

struct KernelInfo {
  void (*fn)(SplitParams);
  size_t smem;
  int tile;
  int threads;
};

template <typename T, int D, int G, class V, bool PAGED>
KernelInfo make_info() {
  using C = SplitCfg<T, D, G, V>;
  return KernelInfo{&split_kv_decode_kernel<T, D, G, V, PAGED>, sizeof(SplitSmem<C>), C::TILE, C::THREADS};
}

// The instance for group size G (1, 2, 4 or 8) of one (T, V, D, PAGED); false for any other G.
template <typename T, class V, int D, bool PAGED>
bool split_instance(int G, KernelInfo* ki);

template <> bool split_instance<__nv_bfloat16, LongTiles, 64, false>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, LongTiles, 64, true>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, LongTiles, 128, false>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, LongTiles, 128, true>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 64, false>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 64, true>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 128, false>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 128, true>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 64, false>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 64, true>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 128, false>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 128, true>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 64, false>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 64, true>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 128, false>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 128, true>(int, KernelInfo*);

}  // namespace ta
