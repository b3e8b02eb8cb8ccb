// Status plumbing shared by the C ABI translation units: a thread-local
// message for pa_last_error() and a helper that records it.
#pragma once

#include "pagedattn.h"

namespace pa {

// Record msg as this thread's last error and return st.
pa_status fail(pa_status st, const char* msg);

}  // namespace pa
