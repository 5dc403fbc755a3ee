// Runtime pieces of libfk: status text, per-(device, stream) workspaces,
// launch accounting and event-based phase timing.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "fk_internal.h"

namespace fk {

namespace {
thread_local std::string g_last_error;
std::mutex g_mu;
std::map<std::pair<int, cudaStream_t>, Workspace *> g_ws;
std::atomic<long long> g_launches{0};

std::mutex g_prof_mu;
int g_prof_level = 0;  // 0 off, 1 every phase, 2 assign + whole update
std::vector<cudaEvent_t> g_event_pool;  // recorded events are reused, not recreated
struct Pending {
  cudaEvent_t a, b;
  int phase;
};
std::vector<Pending> g_pending;
double g_ms[PH_COUNT] = {0, 0, 0, 0, 0};
long long g_assign_launches = 0, g_update_calls = 0, g_prof_launches = 0;
// level 3: per-chunk events of the streamed pipeline (copy begin / end on the
// copy stream, compute begin / end on the compute stream)
struct ChunkEvents {
  cudaEvent_t ev[4];
  long long chunk;
  int buf;
};
std::vector<ChunkEvents> g_chunks;
constexpr size_t kMaxTimelineChunks = 1 << 16;  // 4 events each; recording stops here until read
}  // namespace

int set_error(int status, const std::string &msg) {
  g_last_error = msg;
  return status;
}

int cuda_status(cudaError_t e, const char *what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  if (e == cudaErrorMemoryAllocation) return FK_ENOMEM;
  return FK_ECUDA;
}

int ensure_zeroed(DevBuf &b, size_t bytes, cudaStream_t s) {
  const size_t had = b.bytes;  // a new allocation always changes the size (it only grows)
  FK_TRY(ensure(b, bytes));
  if (b.bytes != had) FK_CUDA(cudaMemsetAsync(b.p, 0, b.bytes, s));
  return FK_OK;
}

int ensure(DevBuf &b, size_t bytes) {
  if (bytes == 0) bytes = 16;
  if (b.bytes >= bytes) return FK_OK;
  if (fault_hit(FK_FAULT_ALLOC))
    return set_error(FK_ENOMEM, "injected allocation failure (FK_FAULT)");
  if (b.p) {
    FK_CUDA(cudaFree(b.p));
    b.p = nullptr;
    b.bytes = 0;
  }
  size_t want = bytes + bytes / 8;  // headroom for small growth
  cudaError_t e = cudaMalloc(&b.p, want);
  if (e != cudaSuccess) {
    b.p = nullptr;
    e = cudaMalloc(&b.p, bytes);
    if (e != cudaSuccess) {
      b.p = nullptr;
      (void)cudaGetLastError();
      return set_error(FK_ENOMEM, "device workspace allocation of " + std::to_string(bytes) + " bytes failed");
    }
    want = bytes;
  }
  b.bytes = want;
  return FK_OK;
}

int set_smem_limit(const void *func, int bytes) {
  // the attribute belongs to the kernel as loaded on the current device
  static std::mutex mu;
  static std::set<std::pair<int, const void *>> done;
  int dev = 0;
  FK_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({dev, func})) return FK_OK;
  FK_CUDA(cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done.insert({dev, func});
  return FK_OK;
}

int workspace_for(cudaStream_t s, Workspace **out) {
  int dev = 0;
  FK_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(dev, s);
  auto it = g_ws.find(key);
  if (it != g_ws.end()) {
    *out = it->second;
    return FK_OK;
  }
  Workspace *ws = new Workspace();
  ws->device = dev;
  ws->stream = s;
  cudaError_t e = cudaMalloc(&ws->err, 16);
  if (e == cudaSuccess) e = cudaMemset(ws->err, 0, 16);
  if (e == cudaSuccess) ws->maxshift = reinterpret_cast<unsigned *>(ws->err + 1);
  if (e == cudaSuccess) e = cudaMallocHost(&ws->h_maxshift, 16);
  if (e != cudaSuccess) {
    if (ws->err) cudaFree(ws->err);
    delete ws;
    return cuda_status(e, "workspace setup");
  }
  g_ws[key] = ws;
  *out = ws;
  return FK_OK;
}

static void free_buf(DevBuf &b) {
  if (b.p) cudaFree(b.p);
  b.p = nullptr;
  b.bytes = 0;
}

int release_device_workspaces() {
  int dev = 0;
  FK_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto it = g_ws.begin(); it != g_ws.end();) {
    if (it->first.first != dev) {
      ++it;
      continue;
    }
    Workspace *ws = it->second;
    DevBuf *bufs[] = {&ws->cn, &ws->ch, &ws->sums, &ws->first, &ws->counts, &ws->offsets,
                      &ws->table, &ws->digit_off, &ws->kv, &ws->x3, &ws->c3, &ws->keys64, &ws->keys_b,
                      &ws->vals_b, &ws->xres, &ws->init_dev, &ws->ids_dev, &ws->centers_dev,
                      &ws->chunk[0], &ws->chunk[1], &ws->gsum, &ws->gcounts, &ws->xn, &ws->ids_alt};
    for (DevBuf *b : bufs) free_buf(*b);
    if (ws->err) cudaFree(ws->err);
    if (ws->h_maxshift) cudaFreeHost(ws->h_maxshift);
    if (ws->copy_stream) cudaStreamDestroy(ws->copy_stream);
    for (int i = 0; i < 2; ++i) {
      if (ws->ready[i]) cudaEventDestroy(ws->ready[i]);
      if (ws->freed[i]) cudaEventDestroy(ws->freed[i]);
    }
    if (ws->shift_ev) cudaEventDestroy(ws->shift_ev);
    delete ws;
    it = g_ws.erase(it);
  }
  return FK_OK;
}

// ---- host-side fault injection (tests of the error paths; no GPU is faulted)
namespace {
std::mutex g_fault_mu;
std::atomic<int> g_fault_kind{-1};  // -1: FK_FAULT not read yet
long long g_fault_left = 0;         // occurrences of the kind still to pass, the last fires

int fault_kind_of(const std::string &name) {
  if (name == "alloc") return FK_FAULT_ALLOC;
  if (name == "h2d") return FK_FAULT_H2D;
  if (name == "launch") return FK_FAULT_LAUNCH;
  return FK_FAULT_NONE;
}

// FK_FAULT=alloc|h2d|launch[:n] arms one failure at the n-th occurrence (default 1).
void read_fault_env() {
  int kind = FK_FAULT_NONE;
  long long nth = 1;
  if (const char *e = getenv("FK_FAULT")) {
    std::string v(e);
    const size_t colon = v.find(':');
    kind = fault_kind_of(v.substr(0, colon));
    if (colon != std::string::npos) nth = atoll(v.c_str() + colon + 1);
  }
  g_fault_left = nth > 0 ? nth : 1;
  g_fault_kind.store(kind);
}
}  // namespace

bool fault_hit(int kind) {
  int k = g_fault_kind.load(std::memory_order_relaxed);
  if (k == FK_FAULT_NONE) return false;
  std::lock_guard<std::mutex> lk(g_fault_mu);
  if (g_fault_kind.load() < 0) read_fault_env();
  if (g_fault_kind.load() != kind) return false;
  if (--g_fault_left > 0) return false;
  g_fault_kind.store(FK_FAULT_NONE);  // fires once
  return true;
}

int set_fault(int kind, long long nth) {
  if (kind < FK_FAULT_NONE || kind > FK_FAULT_LAUNCH || nth < 1)
    return set_error(FK_EINVAL, "fault kind must be FK_FAULT_NONE..FK_FAULT_LAUNCH and nth >= 1");
  std::lock_guard<std::mutex> lk(g_fault_mu);
  g_fault_left = nth;
  g_fault_kind.store(kind);
  return FK_OK;
}

int launched(int n) {
  g_launches.fetch_add(n, std::memory_order_relaxed);
  if (g_prof_level) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_launches += n;
  }
  if (fault_hit(FK_FAULT_LAUNCH)) return set_error(FK_ECUDA, "injected launch failure (FK_FAULT)");
  return FK_OK;
}

long long launch_count() { return g_launches.load(); }

namespace {
cudaEvent_t take_event() {
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_event_pool.empty()) {
      cudaEvent_t e = g_event_pool.back();
      g_event_pool.pop_back();
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}
}  // namespace

PhaseTimer::PhaseTimer(int ph, cudaStream_t st) : phase(ph), s(st) {
  if (!g_prof_level) return;
  if (g_prof_level >= 2 && ph != PH_ASSIGN && ph != PH_UPDATE) return;
  a = take_event();
  b = take_event();
  if (!a || !b) {
    a = b = nullptr;
    return;
  }
  cudaEventRecord(a, s);
}

PhaseTimer::~PhaseTimer() {
  if (!a) return;
  cudaEventRecord(b, s);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_pending.push_back({a, b, phase});
  if (phase == PH_ASSIGN) ++g_assign_launches;
}

void note_update_call() {
  if (!g_prof_level) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  ++g_update_calls;
}

int profile_enable(int on) {
  if (on < 0 || on > 3) return set_error(FK_EINVAL, "profile level must be 0, 1, 2 or 3");
  g_prof_level = on;
  return FK_OK;
}

bool timeline_on() { return g_prof_level == 3; }

int chunk_event(int which, long long chunk, int buf, cudaStream_t s) {
  if (g_prof_level != 3) return FK_OK;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (which == 0) {
    if (g_chunks.size() >= kMaxTimelineChunks) return FK_OK;  // the record is full until read
    ChunkEvents c;
    c.chunk = chunk;
    c.buf = buf;
    for (auto &e : c.ev) FK_CUDA(cudaEventCreate(&e));
    for (auto &e : c.ev) FK_CUDA(cudaEventRecord(e, s));  // a chunk cut short still has four events
    g_chunks.push_back(c);
    return FK_OK;
  }
  // profiling turned on in the middle of a chunk, or a full record: not recorded
  if (g_chunks.empty() || g_chunks.back().chunk != chunk) return FK_OK;
  FK_CUDA(cudaEventRecord(g_chunks.back().ev[which], s));
  return FK_OK;
}

int profile_timeline(double *out, int max_chunks, int *rows) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int n = 0;
  float t0 = 0.f;
  for (size_t i = 0; i < g_chunks.size(); ++i) {
    auto &c = g_chunks[i];
    FK_CUDA(cudaEventSynchronize(c.ev[3]));
    if (out && n < max_chunks) {
      double *row = out + 6 * (size_t)n;
      row[0] = (double)c.chunk;
      row[1] = (double)c.buf;
      for (int k = 0; k < 4; ++k) {
        float ms = 0.f;
        FK_CUDA(cudaEventElapsedTime(&ms, g_chunks[0].ev[0], c.ev[k]));
        row[2 + k] = ms - t0;
      }
      ++n;
    }
  }
  for (auto &c : g_chunks)
    for (auto &e : c.ev) cudaEventDestroy(e);
  g_chunks.clear();
  *rows = n;
  return FK_OK;
}

int profile_read(fk_profile *out, int reset) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto &p : g_pending) {
    float ms = 0.f;
    cudaEventSynchronize(p.b);
    if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) g_ms[p.phase] += ms;
    g_event_pool.push_back(p.a);
    g_event_pool.push_back(p.b);
  }
  g_pending.clear();
  if (out) {
    out->assign_ms = g_ms[PH_ASSIGN];
    out->sort_ms = g_ms[PH_SORT];
    out->reduce_ms = g_ms[PH_REDUCE];
    out->finalize_ms = g_ms[PH_FINALIZE];
    out->update_ms = g_ms[PH_UPDATE];
    out->assign_launches = g_assign_launches;
    out->update_calls = g_update_calls;
    out->kernel_launches = g_prof_launches;
  }
  if (reset) {
    for (double &v : g_ms) v = 0;
    g_assign_launches = g_update_calls = g_prof_launches = 0;
  }
  return FK_OK;
}

size_t esize(int dtype) { return dtype == FK_F32 ? 4 : 2; }

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

const char *last_error() { return g_last_error.c_str(); }

}  // namespace fk
