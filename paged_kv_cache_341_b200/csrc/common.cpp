// Per-thread last-error message of libpagedattn.so.
#include "pa_common.h"

namespace {
thread_local std::string g_last_error;
}

namespace pa {

pa_status fail(pa_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

pa_status ok() {
  g_last_error.clear();
  return PA_OK;
}

}  // namespace pa

extern "C" const char* pa_last_error(void) { return g_last_error.c_str(); }
