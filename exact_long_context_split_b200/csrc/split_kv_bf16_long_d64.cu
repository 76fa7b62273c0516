// Split-KV decode kernel instances: bf16 K/V, LongTiles, head_dim 64.
#define TA_INST_T __nv_bfloat16
#define TA_INST_V LongTiles
#define TA_INST_D 64
#define TA_INST_PAGED false
#include "split_kv_instance.cuh"
