// Internal helpers shared by the C-ABI translation units (not exported).
#pragma once

#include <string>

#include "srnl_scan.h"

namespace srnl {

// Same validation srnl_scan_create applies; sets the calling thread's error.
srnl_status validate_scan_config(const srnl_scan_config* cfg);

// Record a message for srnl_scan_last_error(NULL) on the calling thread.
void set_thread_error(const std::string& msg);

}  // namespace srnl
