// Bits of the device error word (mapped to tt_status_t by the host).
#pragma once
namespace tt {
constexpr unsigned kErrDeviceArg = 1u;  // ctx_lens[n] outside [0, capacity]
constexpr unsigned kErrTimeout = 2u;    // a bounded in-kernel wait gave up
constexpr unsigned kErrInternal = 4u;   // a kernel found its launch unusable (e.g. shared-memory alignment)
}  // namespace tt
