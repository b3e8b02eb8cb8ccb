#include "status.h"

#include <cstdio>
#include <cstring>

namespace {
thread_local char g_last_error[512] = "";
}

namespace pa {

pa_status fail(pa_status st, const char* msg) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s", msg ? msg : "");
  return st;
}

}  // namespace pa

extern "C" {

const char* pa_last_error(void) { return g_last_error; }

const char* pa_status_string(int32_t status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_OUT_OF_BOUNDS: return "PA_ERR_OUT_OF_BOUNDS";
    case PA_ERR_NO_FREE_BLOCKS: return "PA_ERR_NO_FREE_BLOCKS";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
    default: return "PA_STATUS_UNKNOWN";
  }
}

}  // extern "C"
