// Split-KV decode kernel instances over a paged cache: f32 K/V, LongTiles, head_dim 128.
#define TA_INST_T float
#define TA_INST_V LongTiles
#define TA_INST_D 128
#define TA_INST_PAGED true
#include "split_kv_instance.cuh"
