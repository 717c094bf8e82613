// abi_internal.h -- helpers of the C ABI shared by its translation units
// (internal; not part of the public header).
#pragma once

#include "../../include/strata_moe.h"

// Record a formatted message as the thread's last error and return s.
strata_status strata_set_error(strata_status s, const char *fmt, ...);
// Check a layer descriptor; on failure the reason is the last error.
strata_status strata_check_desc(const strata_moe_desc *desc);
