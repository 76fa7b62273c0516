// Body of one split-KV instance translation unit: defines split_instance<T, V, D, PAGED> for
// the TA_INST_T / TA_INST_V / TA_INST_D / TA_INST_PAGED the including file sets, over every
// group size.
#pragma once
#include "split_kv_instances.h"

namespace ta {

template <>
bool split_instance<TA_INST_T, TA_INST_V, TA_INST_D, TA_INST_PAGED>(int G, KernelInfo* ki) {
  switch (G) {
    case 1: *ki = make_info<TA_INST_T, TA_INST_D, 1, TA_INST_V, TA_INST_PAGED>(); return true;
    case 2: *ki = make_info<TA_INST_T, TA_INST_D, 2, TA_INST_V, TA_INST_PAGED>(); return true;
    case 4: *ki = make_info<TA_INST_T, TA_INST_D, 4, TA_INST_V, TA_INST_PAGED>(); return true;
    case 8: *ki = make_info<TA_INST_T, TA_INST_D, 8, TA_INST_V, TA_INST_PAGED>(); return true;
    default: return false;
  }
}

}  // namespace ta
