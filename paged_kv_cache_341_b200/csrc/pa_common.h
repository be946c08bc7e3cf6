// Shared host-side helpers of libpagedattn.so: status + per-thread message.
#ifndef PAGEDATTN_PA_COMMON_H
#define PAGEDATTN_PA_COMMON_H

#include <string>

#include "pa.h"

namespace pa {

// Record `msg` as this thread's last error and return `st`.
pa_status fail(pa_status st, const std::string& msg);
// Clear this thread's last error and return PA_OK.
pa_status ok();

}  // namespace pa

#endif
