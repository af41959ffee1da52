// Host-side helpers of capi.cu shared with the other C-ABI translation units (internal).
#pragma once
#include <string>
#include <vector>

#include "../../include/tp.h"

namespace tp {

struct IrrepTerm {
  int mul, l, parity;   // parity +1 (e) or -1 (o)
};

// Parses "32x0e+32x1o" into terms; false with a reason on a syntax error.
bool parse_irreps_terms(const char* s, std::vector<IrrepTerm>& out, std::string& why);

// Records the thread's message for tp_last_error_message and returns st.
tp_status_t set_failure(tp_status_t st, const std::string& msg);

// The per-device error word of calls without index checks (code 6: a bounded wait gave up).
int* device_error_ptr();

}  // namespace tp
