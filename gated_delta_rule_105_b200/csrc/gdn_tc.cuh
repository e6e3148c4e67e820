// tcgen05 (5th-generation tensor core) chunked forward kernel for bf16 inputs.
#pragma once

#include "gdn_common.cuh"

namespace gdn {

inline bool tc_supported(const FwdParams&, bool, bool) { return false; }
inline const char* tc_last_error() { return "tcgen05 kernel not built"; }
inline gdn_status launch_tc(const FwdParams&, bool, bool, unsigned*, cudaStream_t) { return GDN_ERR_UNSUPPORTED; }

}  // namespace gdn
