// What the library asks of the current device, queried once per device and
// cached: its SM count (the plans' wave sizes) and how many thread-block
// clusters of a given shape it holds at once (the cluster kernels' head
// limits).
#pragma once

#include <cstddef>

namespace la {

// SMs of the current device. When no device can be queried (sizing a
// workspace on a machine without a GPU), the 148 SMs of a full B200.
int device_sms();

// Most clusters of `cluster` CTAs that the current device holds at once
// when each CTA has `threads` threads and `smem` bytes of dynamic shared
// memory and no register or TMEM limit binds: the occupancy of a plain
// kernel of that shape (cudaOccupancyMaxActiveClusters). 0 if the query fails.
int max_active_clusters(int cluster, int threads, size_t smem);

}  // namespace la
