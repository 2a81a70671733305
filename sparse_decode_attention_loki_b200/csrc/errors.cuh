// Device-side error count: timeouts of the kernels' bounded waits.  Each
// translation unit of the library holds its own counter; the host sums them
// (loki_device_error_count).
#pragma once

namespace loki {

static __device__ unsigned int g_loki_device_errors;

}  // namespace loki
