// Library-internal state shared by its translation units (kept in capi.cu):
// the per-device status word that bounded waits report into, the wait limit,
// the debug flags, the SM count, and the host-side block-mask check.
#pragma once

#include <cstdint>

#include "../../include/sparse_attn.h"

namespace sa {

int device_status_word(int32_t** out);  // SA_OK or SA_ERR_CUDA
long long wait_limit_cycles();
int32_t debug_flags();                  // as set by sparse_attn_set_debug
int device_sm_count();                  // 0 when the query fails

// A block mask in host memory with T tiles per side is well formed: every
// count in [0, T], each row's listed tiles strictly ascending inside [0, T),
// full flags 0 or 1.  SA_OK or SA_ERR_INVALID_ARG; O(T^2).
int check_host_mask(const sa_block_mask* m, int64_t T);

// The arrays of a block mask that a kernel reads are readable by the current
// device: its own memory, managed memory or pinned host memory (pageable host
// memory or another device's memory would fault the kernel).  SA_OK,
// SA_ERR_INVALID_ARG, or SA_ERR_CUDA when the device query fails.
int check_device_mask(const sa_block_mask* m);

}  // namespace sa
