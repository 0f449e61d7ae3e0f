// Expert staging without a host round trip per layer: the in-stream
// doorbell of the "Betelgeuse" post (a kernel in the decode stream rings a
// mapped host flag only when a layer misses; a host pager fills the slots;
// the stream goes on once they are filled).
//
// Per layer, on the compute stream (all capturable in a CUDA graph):
//   moe_slot_resolve -> moe_miss_post -> moe_wait_done -> expert FFN
// moe_miss_post takes the next request number from a device counter.  With
// misses it writes the miss list and then the number into a mailbox in
// mapped pinned host memory (the doorbell); without misses it marks the
// request done in a device word itself.  moe_wait_done holds the stream
// until either done word reaches the request number, bounded by
// %globaltimer (MOE_ERR_TIMEOUT).  The stager is a host thread: it polls
// the mailbox, copies each missed blob from its pinned host copy into the
// victim slot on the caller's copy streams (half a blob per copy), waits for
// the copies on the host and then writes the request number into the
// mailbox's done word.  Nothing the stager does needs a compute queue: a
// kernel or stream operation of its own could sit behind the launches that
// the wait holds up (streams share hardware queues), which would deadlock
// until the wait's bound.
//
// Ordering: a request with misses is posted only after the previous
// request's wait has passed, i.e. after the stager has read the previous
// mailbox contents, so the mailbox is never rewritten while the stager may
// read it; requests without misses never touch the mailbox.  Both done
// words only grow: the stager handles requests in order, and the device
// marks a request without misses after every earlier one is done.
#include <atomic>
#include <chrono>
#include <thread>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
namespace {

// Mailbox layout (host-mapped): header words, then the miss lists.
constexpr int MB_SEQ = 0, MB_LAYER = 1, MB_N = 2, MB_DONE = 3, MB_HDR = 4;
constexpr int MB_MAXM = 1024;   // misses per request (T*k <= 1024)

__global__ void miss_post_kernel(const int32_t* n_miss,
                                 const int32_t* miss_expert,
                                 const int32_t* miss_slot, int P, int layer,
                                 int slot_base, int32_t* mb,
                                 uint32_t* sync, int32_t* err) {
  __shared__ uint32_t s_seq;
  __shared__ int s_n;
  if (threadIdx.x == 0) {
    const uint32_t seq = sync[0] + 1u;   // stream-ordered: plain update
    sync[0] = seq;
    int n = *n_miss;
    if (n < 0 || n > P) {
      set_err(err, MOE_ERR_DEVICE);
      n = 0;
    }
    s_seq = seq;
    s_n = n;
    if (n == 0) {   // nothing to stage: the request is done at once
      __threadfence();
      *reinterpret_cast<volatile uint32_t*>(sync + 1) = seq;
    }
  }
  __syncthreads();
  const int n = s_n;
  if (n == 0) return;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    mb[MB_HDR + i] = miss_expert[i];
    mb[MB_HDR + MB_MAXM + i] = slot_base + miss_slot[i];
  }
  if (threadIdx.x == 0) {
    mb[MB_LAYER] = layer;
    mb[MB_N] = n;
  }
  // the list reaches host memory before the request number does
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    *reinterpret_cast<volatile uint32_t*>(mb + MB_SEQ) = s_seq;
  }
}

__global__ void wait_done_kernel(const int32_t* mb, const uint32_t* sync,
                                 uint32_t timeout_us, int32_t* err) {
  const uint32_t target =
      *reinterpret_cast<const volatile uint32_t*>(sync);
  const uint64_t t0 = globaltimer();
  for (;;) {
    uint32_t d, h;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                 : "=r"(d) : "l"(sync + 1) : "memory");
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];"
                 : "=r"(h) : "l"(mb + MB_DONE) : "memory");
    if ((int32_t)(d - target) >= 0 || (int32_t)(h - target) >= 0) return;
    if (globaltimer() - t0 > (uint64_t)timeout_us * 1000ull) {
      set_err(err, MOE_ERR_TIMEOUT);
      return;
    }
    __nanosleep(200);
  }
}

}  // namespace

bool is_device_memory(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

// The host pager.
struct Stager {
  volatile int32_t* mb = nullptr;
  uint32_t last = 0;   // the mailbox's request number when created
  uint8_t* pool = nullptr;
  int64_t stride = 0, blob = 0;
  std::vector<const uint8_t*> src;   // [L * E] pinned host blobs
  int L = 0, E = 0, dev = 0;
  std::vector<cudaStream_t> cs;
  std::vector<cudaEvent_t> ev;
  std::thread th;
  std::atomic<bool> stop{false};
  std::atomic<int> status{MOE_OK};
  std::atomic<long long> requests{0}, copies{0};

  void run() {
    cudaSetDevice(dev);
    int idle = 0;
    const int64_t half = ((blob / 2) + 255) / 256 * 256;
    while (!stop.load(std::memory_order_relaxed)) {
      const uint32_t seq = (uint32_t)mb[MB_SEQ];
      if (seq == last) {
        if (++idle > 2048) std::this_thread::yield();
        continue;
      }
      idle = 0;
      std::atomic_thread_fence(std::memory_order_acquire);
      last = seq;
      const int layer = mb[MB_LAYER], n = mb[MB_N];
      int j = 0;
      bool bad = n < 0 || n > MB_MAXM || layer < 0 || layer >= L;
      for (int i = 0; !bad && i < n; ++i) {
        const int e = mb[MB_HDR + i], slot = mb[MB_HDR + MB_MAXM + i];
        if (e < 0 || e >= E || slot < 0 || !src[(size_t)layer * E + e]) {
          status.store(MOE_ERR_CAPACITY);   // no host copy of this blob
          continue;
        }
        const uint8_t* from = src[(size_t)layer * E + e];
        uint8_t* to = pool + (int64_t)slot * stride;
        for (int64_t a = 0; a < blob; a += half, ++j) {
          const int64_t b = a + half < blob ? a + half : blob;
          if (cudaMemcpyAsync(to + a, from + a, (size_t)(b - a),
                              cudaMemcpyHostToDevice,
                              cs[j % cs.size()]) != cudaSuccess)
            status.store(MOE_ERR_CUDA);
        }
        copies.fetch_add(1);
      }
      if (bad) status.store(MOE_ERR_INVALID);
      // wait for the copies here, then raise the done word
      const size_t used = (size_t)j < cs.size() ? (size_t)j : cs.size();
      for (size_t k = 0; k < used; ++k)
        if (cudaEventRecord(ev[k], cs[k]) != cudaSuccess)
          status.store(MOE_ERR_CUDA);
      for (size_t k = 0; k < used; ++k)
        if (cudaEventSynchronize(ev[k]) != cudaSuccess)
          status.store(MOE_ERR_CUDA);
      std::atomic_thread_fence(std::memory_order_release);
      mb[MB_DONE] = (int32_t)seq;
      requests.fetch_add(1);
    }
  }
};

}  // namespace moe

using moe::Stager;

extern "C" size_t moe_mailbox_bytes(void) {
  return (size_t)(moe::MB_HDR + 2 * moe::MB_MAXM) * 4;
}

extern "C" moe_status moe_miss_post(const int32_t* n_miss,
                                    const int32_t* miss_expert,
                                    const int32_t* miss_slot, int P,
                                    int layer, int slot_base, void* mailbox,
                                    uint32_t* sync, int32_t* err,
                                    void* stream) {
  if (!n_miss || !miss_expert || !miss_slot || !mailbox || !sync)
    return MOE_ERR_INVALID;
  if (P < 1 || P > moe::MB_MAXM || layer < 0 || slot_base < 0)
    return MOE_ERR_SHAPE;
  // the mailbox must be mapped pinned host memory and sync device memory:
  // checked here so that a wrong pointer is an argument error, not a fault
  void* mb_dev = nullptr;
  if (cudaHostGetDevicePointer(&mb_dev, mailbox, 0) != cudaSuccess ||
      !mb_dev) {
    cudaGetLastError();
    return MOE_ERR_INVALID;
  }
  if (!moe::is_device_memory(sync)) return MOE_ERR_INVALID;
  moe::miss_post_kernel<<<1, 128, 0, (cudaStream_t)stream>>>(
      n_miss, miss_expert, miss_slot, P, layer, slot_base,
      static_cast<int32_t*>(mb_dev), sync, err);
  return moe::launch_status();
}

extern "C" moe_status moe_wait_done(void* mailbox, const uint32_t* sync,
                                    uint32_t timeout_us, int32_t* err,
                                    void* stream) {
  if (!mailbox || !sync || !err || timeout_us == 0) return MOE_ERR_INVALID;
  void* mb_dev = nullptr;
  if (cudaHostGetDevicePointer(&mb_dev, mailbox, 0) != cudaSuccess ||
      !mb_dev) {
    cudaGetLastError();
    return MOE_ERR_INVALID;
  }
  if (!moe::is_device_memory(sync) || !moe::is_device_memory(err))
    return MOE_ERR_INVALID;
  moe::wait_done_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(
      static_cast<const int32_t*>(mb_dev), sync, timeout_us, err);
  return moe::launch_status();
}

extern "C" moe_status moe_stager_create(void** out, void* mailbox,
                                        uint8_t* pool,
                                        int64_t blob_stride,
                                        int64_t blob_bytes,
                                        const void* const* host_blob, int L,
                                        int E, void* const* copy_streams,
                                        int n_copy_streams) {
  if (!out || !mailbox || !pool || !host_blob || !copy_streams)
    return MOE_ERR_INVALID;
  if (L < 1 || E < 1 || n_copy_streams < 1 || blob_bytes < 1 ||
      blob_stride < blob_bytes)
    return MOE_ERR_SHAPE;
  void* mb_dev = nullptr;
  if (cudaHostGetDevicePointer(&mb_dev, mailbox, 0) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_INVALID;   // the mailbox is not mapped pinned memory
  }
  if (!moe::is_device_memory(pool)) return MOE_ERR_INVALID;
  auto* st = new Stager;
  st->mb = static_cast<volatile int32_t*>(mailbox);
  // requests posted from now on are the stager's (read before the thread
  // starts, so a post that comes before the thread runs is not lost)
  st->last = (uint32_t)st->mb[moe::MB_SEQ];
  st->pool = pool;
  st->stride = blob_stride;
  st->blob = blob_bytes;
  st->L = L;
  st->E = E;
  st->src.assign(reinterpret_cast<const uint8_t* const*>(host_blob),
                 reinterpret_cast<const uint8_t* const*>(host_blob) +
                     (size_t)L * E);
  for (int i = 0; i < n_copy_streams; ++i)
    st->cs.push_back((cudaStream_t)copy_streams[i]);
  st->ev.resize(n_copy_streams);
  if (cudaGetDevice(&st->dev) != cudaSuccess) {
    delete st;
    return MOE_ERR_CUDA;
  }
  for (auto& e : st->ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      delete st;
      return MOE_ERR_CUDA;
    }
  st->th = std::thread([st] { st->run(); });
  *out = st;
  return MOE_OK;
}

extern "C" moe_status moe_stager_stats(void* stager, int64_t* requests,
                                       int64_t* copies) {
  if (!stager) return MOE_ERR_INVALID;
  auto* st = static_cast<Stager*>(stager);
  if (requests) *requests = st->requests.load();
  if (copies) *copies = st->copies.load();
  return (moe_status)st->status.load();
}

extern "C" moe_status moe_stager_destroy(void* stager) {
  if (!stager) return MOE_ERR_INVALID;
  auto* st = static_cast<Stager*>(stager);
  st->stop.store(true);
  if (st->th.joinable()) st->th.join();
  for (auto s : st->cs) cudaStreamSynchronize(s);
  for (auto e : st->ev)
    if (e) cudaEventDestroy(e);
  const moe_status r = (moe_status)st->status.load();
  delete st;
  return r;
}
