// Host-side decisions about the buffers and budgets handed to the library: whether the current GPU can
// address a buffer (and with which address), whether byte ranges overlap, and how a wait budget in
// nanoseconds becomes a budget in SM clock cycles.
//
// The functions take the CUDA runtime's pointer-attribute record and a table of the two peer-access calls
// as inputs, so a plain C++ test can drive every decision with fabricated attributes and a stand-in for
// the runtime (no GPU needed).
#pragma once

#include <cuda_runtime_api.h>
#include <stddef.h>
#include <stdint.h>

#include "lvsa.h"

namespace lvsa {

// Device-side waits count SM clock cycles; a budget in ns is converted at 2 GHz (at lower clocks the wait
// lasts longer in wall time, never shorter).
constexpr double kBudgetCyclesPerNs = 2.0;
// Largest accepted wait budget: 1000 s (2e12 cycles, far from the range of the signed 64-bit counter).
constexpr unsigned long long kMaxWaitBudgetNs = 1000000000000ull;
constexpr unsigned long long kMinWaitBudgetNs = 1000ull;

// Cycles for a budget already checked against [kMinWaitBudgetNs, kMaxWaitBudgetNs].
inline long long wait_budget_cycles(unsigned long long ns) {
  return static_cast<long long>(static_cast<double>(ns) * kBudgetCyclesPerNs);
}

// The runtime calls the addressability decision needs (the library passes the CUDA runtime's own).
struct PeerOps {
  cudaError_t (*can_access)(int* can, int device, int peer);  // cudaDeviceCanAccessPeer
  cudaError_t (*enable)(int peer, unsigned int flags);        // cudaDeviceEnablePeerAccess (current device)
  cudaError_t (*clear_error)();                               // cudaGetLastError
};

// Can device `dev` (the current device) load from and store to the buffer whose attributes are `at`?
//  - its own memory: yes;
//  - another GPU's memory: only where peer access is possible; it is enabled here if it is not yet
//    (enabling it twice is not an error);
//  - host memory that CUDA maps for the device (pinned or registered) and managed memory: yes;
//  - pageable host memory or memory CUDA does not know: no.
// On success *dptr is the address the device uses and *remote is 1 when the buffer is not this GPU's own
// memory (a kernel storing there must release its stores at system scope).  Errors:
// LVSA_ERR_INVALID_ARG (the GPU cannot address the buffer), LVSA_ERR_CUDA (enabling peer access failed).
inline lvsa_status device_address(const cudaPointerAttributes& at, int dev, const PeerOps& ops, void** dptr,
                                  int* remote) {
  if (at.type == cudaMemoryTypeUnregistered || at.devicePointer == nullptr) return LVSA_ERR_INVALID_ARG;
  if (at.type == cudaMemoryTypeDevice && at.device != dev) {
    int can = 0;
    if (ops.can_access(&can, dev, at.device) != cudaSuccess || !can) return LVSA_ERR_INVALID_ARG;
    const cudaError_t e = ops.enable(at.device, 0);
    if (e == cudaErrorPeerAccessAlreadyEnabled) {
      ops.clear_error();  // not sticky, but leave no error behind for the next cudaGetLastError
    } else if (e != cudaSuccess) {
      ops.clear_error();
      return LVSA_ERR_CUDA;
    }
  }
  *dptr = at.devicePointer;
  *remote = (at.type == cudaMemoryTypeDevice && at.device == dev) ? 0 : 1;
  return LVSA_OK;
}

// Byte ranges [a, a + na) and [b, b + nb); an empty range overlaps nothing.
inline bool ranges_disjoint(const void* a, size_t na, const void* b, size_t nb) {
  if (na == 0 || nb == 0) return true;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x + na <= y || y + nb <= x;
}

}  // namespace lvsa
