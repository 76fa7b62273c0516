// Split-KV decode kernel instances: f32 K/V, ShortTiles, head_dim 64.
#define TA_INST_T float
#define TA_INST_V ShortTiles
#define TA_INST_D 64
#define TA_INST_PAGED false
#include "split_kv_instance.cuh"
