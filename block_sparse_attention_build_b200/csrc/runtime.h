// Library-internal state shared by its translation units (kept in capi.cu):
// the per-device status word that bounded waits report into, the wait limit,
// and the SM count.
#pragma once

#include <cstdint>

namespace sa {

int device_status_word(int32_t** out);  // SA_OK or SA_ERR_CUDA
long long wait_limit_cycles();
int device_sm_count();                  // 0 when the query fails

}  // namespace sa
