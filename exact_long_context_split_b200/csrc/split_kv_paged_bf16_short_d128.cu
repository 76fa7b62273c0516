// Split-KV decode kernel instances over a paged cache: bf16 K/V, ShortTiles, head_dim 128.
#define TA_INST_T __nv_bfloat16
#define TA_INST_V ShortTiles
#define TA_INST_D 128
#define TA_INST_PAGED true
#include "split_kv_instance.cuh"
