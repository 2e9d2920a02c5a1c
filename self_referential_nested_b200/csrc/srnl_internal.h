// Internal helpers shared by the C-ABI translation units (not exported).
#pragma once

#include <cuda_runtime.h>

#include <string>

#include "srnl_scan.h"

namespace srnl {

// Same validation srnl_scan_create applies; sets the calling thread's error.
srnl_status validate_scan_config(const srnl_scan_config* cfg);

// Record a message for srnl_scan_last_error(NULL) on the calling thread.
void set_thread_error(const std::string& msg);

// One thread waits (bounded, limit_ns of wall time) on an mbarrier that nothing completes and
// writes SRNL_E_TIMEOUT, or SRNL_OK had the wait completed, to the device int *status.
cudaError_t launch_wait_probe(unsigned long long limit_ns, int* status, cudaStream_t s);

}  // namespace srnl
