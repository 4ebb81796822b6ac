// Identity of the calling thread's current CUDA context, for host caches that
// hold per-context state (a symbol's device address, a kernel's shared-memory
// opt-in): after cudaDeviceReset the device's next context is a new one and
// such state must be set up again.
#pragma once

namespace h3rr {

// Process-unique id of the current context (ids are never reused, unlike
// context handles); false if no context is current or the driver cannot say.
bool current_context_id(unsigned long long* id);

}  // namespace h3rr
