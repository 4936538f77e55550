// Drives the library's host-side buffer decisions (block_sparse_attention_frame_b200/csrc/buffer_checks.h)
// with fabricated CUDA pointer attributes and a stand-in for the peer-access calls: no GPU, no CUDA
// runtime linked.  Prints one line per case; the pytest wrapper compares them.
#include <cstdio>

#include "buffer_checks.h"

namespace {
int g_can = 1;                               // cudaDeviceCanAccessPeer answer
cudaError_t g_enable = cudaSuccess;          // cudaDeviceEnablePeerAccess result
int g_enable_calls = 0, g_clear_calls = 0;

cudaError_t fake_can(int* can, int, int) { *can = g_can; return cudaSuccess; }
cudaError_t fake_can_fails(int* can, int, int) { *can = 0; return cudaErrorInvalidDevice; }
cudaError_t fake_enable(int, unsigned int) { ++g_enable_calls; return g_enable; }
cudaError_t fake_clear() { ++g_clear_calls; return cudaSuccess; }

cudaPointerAttributes attrs(cudaMemoryType type, int device, void* dptr) {
  cudaPointerAttributes a{};
  a.type = type;
  a.device = device;
  a.devicePointer = dptr;
  a.hostPointer = nullptr;
  return a;
}

void run(const char* what, const cudaPointerAttributes& a, int dev, const lvsa::PeerOps& ops) {
  void* d = nullptr;
  int remote = -1;
  g_enable_calls = g_clear_calls = 0;
  const lvsa_status s = lvsa::device_address(a, dev, ops, &d, &remote);
  std::printf("%s status=%d ptr=%p remote=%d enable=%d clear=%d\n", what, static_cast<int>(s), d, remote,
              g_enable_calls, g_clear_calls);
}
}  // namespace

int main() {
  void* p = reinterpret_cast<void*>(0x7f0000001000ull);
  const lvsa::PeerOps ops{fake_can, fake_enable, fake_clear};
  run("own", attrs(cudaMemoryTypeDevice, 0, p), 0, ops);
  run("peer", attrs(cudaMemoryTypeDevice, 3, p), 0, ops);
  g_enable = cudaErrorPeerAccessAlreadyEnabled;
  run("peer_enabled", attrs(cudaMemoryTypeDevice, 3, p), 0, ops);
  g_enable = cudaErrorTooManyPeers;
  run("peer_enable_fails", attrs(cudaMemoryTypeDevice, 3, p), 0, ops);
  g_enable = cudaSuccess;
  g_can = 0;
  run("peer_no_access", attrs(cudaMemoryTypeDevice, 3, p), 0, ops);
  g_can = 1;
  run("peer_query_fails", attrs(cudaMemoryTypeDevice, 3, p), 0, lvsa::PeerOps{fake_can_fails, fake_enable, fake_clear});
  run("pinned_host", attrs(cudaMemoryTypeHost, 0, p), 0, ops);
  run("managed", attrs(cudaMemoryTypeManaged, 0, p), 0, ops);
  run("pageable", attrs(cudaMemoryTypeUnregistered, 0, nullptr), 0, ops);
  run("no_device_ptr", attrs(cudaMemoryTypeHost, 0, nullptr), 0, ops);
  // overlap of byte ranges
  char* b = reinterpret_cast<char*>(0x100000);
  std::printf("disjoint %d %d %d %d %d\n", lvsa::ranges_disjoint(b, 16, b + 16, 16),
              lvsa::ranges_disjoint(b, 17, b + 16, 16), lvsa::ranges_disjoint(b + 16, 16, b, 17),
              lvsa::ranges_disjoint(b, 0, b, 16), lvsa::ranges_disjoint(b, 64, b + 8, 8));
  // wait budgets: ns -> SM cycles at 2 GHz, the largest accepted budget stays far inside 64 bits
  std::printf("cycles %lld %lld %lld\n", lvsa::wait_budget_cycles(lvsa::kMinWaitBudgetNs),
              lvsa::wait_budget_cycles(4000000000ull), lvsa::wait_budget_cycles(lvsa::kMaxWaitBudgetNs));
  return 0;
}
