// Internal declarations shared by the host and device translation units of libwq.
#pragma once
#include "../../include/wq.h"

namespace wq {
wq_status set_error(wq_status st, const char* fmt, ...);
wq_status ok();
const char* last_error();
inline bool valid_group(int g) { return g == 32 || g == 64 || g == 128; }
}  // namespace wq
