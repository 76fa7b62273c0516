// Split-KV decode kernel instances: f32 K/V, LongTiles, head_dim 64.
#define TA_INST_T float
#define TA_INST_V LongTiles
#define TA_INST_D 64
#define TA_INST_PAGED false
#include "split_kv_instance.cuh"
