// Per-host-thread count of kernel launches issued by the last public call.
#pragma once

namespace p3d {
extern thread_local int g_launches;
inline void count_launch(int n = 1) { g_launches += n; }
inline void reset_launches() { g_launches = 0; }
}  // namespace p3d
