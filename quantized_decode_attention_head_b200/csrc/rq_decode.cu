// Decode dispatchers: shared-memory sizing, the (head_dim, GQA group)
// dispatch of launches and occupancy queries, and the device scratch array
// of rq_decode_attention_noalloc.  The kernel itself is in rq_decode.cuh.
#include <mutex>

#include "rq_decode.cuh"

namespace rq {

// per-warp scale scratch of the tile path (Cfg<D, G>::SCRATCH floats), at the
// base of the dynamic shared memory
constexpr int scale_scratch_bytes(int D) { return NW * 8 * ((D / 32) * 8 + 4 + (D / 8) * 2 + 4) * 4; }
static_assert(scale_scratch_bytes(128) == NW * Cfg<128, 4>::SCRATCH * 4, "scale scratch layout");
static_assert(scale_scratch_bytes(64) == NW * Cfg<64, 4>::SCRATCH * 4, "scale scratch layout");

// Shared memory of the roles that alias the tile rings (after the scale
// scratch): the merge slots (warp slots + the item partial), the window
// item's two buffers of one K and one V chunk (which start at the base and
// so also cover the scale scratch), and the pack-ahead item's staged K and V
// tile.
int decode_free_bytes(int G, int D) {
  const int part = partial_floats(G, D);
  int merge = (NW + 1) * part * 4;
  const int win = window_smem_bytes(D) - scale_scratch_bytes(D);
  if (merge < win) merge = win;
  const int pack = D == 128 ? (int)sizeof(TileSmem<128>) : (int)sizeof(TileSmem<64>);
  return merge > pack ? merge : pack;
}

int decode_smem_bytes(int n_items, int stages, int stage_bytes, int G, int D) {
  const int ring = NW * stages * stage_bytes;
  const int other = decode_free_bytes(G, D);
  const int need = ring > other ? ring : other;
  return (need + 127) / 128 * 128 + scale_scratch_bytes(D);
}

int decode_resident_ctas(int D, int G, int cluster, int smem, int q_terms) {
#define RQ_DG(DD, GG) \
  if (D == DD && G == GG) return decode_resident_ctas_dg<DD, GG>(cluster, smem, q_terms);
  RQ_DG(128, 1) RQ_DG(128, 2) RQ_DG(128, 4) RQ_DG(128, 8)
  RQ_DG(64, 1) RQ_DG(64, 2) RQ_DG(64, 4) RQ_DG(64, 8)
#undef RQ_DG
  return 1;
}

// Self-test of the device timeout path: one thread waits on an mbarrier that
// nothing ever completes, with the same bounded wait the decode pipeline uses,
// gives up after limit_ns and records the timeout in the status word the way
// a decode kernel does.
__global__ void wait_timeout_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_fence_init();
  if (!mbar_wait_bounded(&bar, 0u, limit_ns)) atomicCAS(status, 0, kDeviceTimeout);
}

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, int smem, cudaStream_t st) {
  const int D = a.g.D, G = a.g.G;
#define RQ_DG(DD, GG) \
  if (D == DD && G == GG) return launch_decode_dg<DD, GG>(a, smem, st);
  RQ_DG(128, 1) RQ_DG(128, 2) RQ_DG(128, 4) RQ_DG(128, 8)
  RQ_DG(64, 1) RQ_DG(64, 2) RQ_DG(64, 4) RQ_DG(64, 8)
#undef RQ_DG
  return cudaErrorInvalidValue;
}

}  // namespace rq

// ---------------------------------------------------------------------------
// Scratch for rq_decode_attention_noalloc: a file-scope device array, so that
// callers that must not allocate device memory (see include/rq.h) can still
// run the split-K decode.  Every device that loads this library holds it
// until the process exits.  Host code may only use the address returned by
// cudaGetSymbolAddress for the current device, never the array's name.
namespace rq {
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

cudaError_t noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // once per device, with that device current
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}
}  // namespace rq
