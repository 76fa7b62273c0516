// Host-side handle of the compiled split-KV kernel instances.  Each (element type, tile
// configuration, head_dim) is compiled in a translation unit of its own
// (split_kv_<type>_<tiles>_d<D>.cu) so that the instances build in parallel.
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

template <typename T, int D, int G, class V>
KernelInfo make_info() {
  using C = SplitCfg<T, D, G, V>;
  return KernelInfo{&split_kv_decode_kernel<T, D, G, V>, sizeof(SplitSmem<C>), C::TILE, C::THREADS};
}

// The instance for group size G (1, 2, 4 or 8) of one (T, V, D); false for any other G.
template <typename T, class V, int D>
bool split_instance(int G, KernelInfo* ki);

template <> bool split_instance<__nv_bfloat16, LongTiles, 64>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, LongTiles, 128>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 64>(int, KernelInfo*);
template <> bool split_instance<__nv_bfloat16, ShortTiles, 128>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 64>(int, KernelInfo*);
template <> bool split_instance<float, LongTiles, 128>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 64>(int, KernelInfo*);
template <> bool split_instance<float, ShortTiles, 128>(int, KernelInfo*);

}  // namespace ta
