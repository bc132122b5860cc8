// pool.cu -- the bounded, top-k-aware LRU pool of expert slots.
//
// "Red Metal dev8 -- resident routed top-k layer", steps 1-3: the
// hard-bounded LRU makes every selected expert resident; selected experts
// are protected from eviction while the remaining misses are filled; every
// selected slot is pinned for the work that uses it.  "Red Lite dev9 --
// native runtime foundation", section "Native selftest": hard capacity
// enforcement, LRU hit/miss/eviction, protection of the current top-k
// during acquire_many, in-flight slot protection.
//
// The policy is host code with no device dependence (redlite_moe_pool_plan,
// testable without a GPU); redlite_moe_pool_acquire adds the data movement:
// the misses' three matrices are copied host -> device into their slots, the
// slot table is updated (an evicted expert's entry is cleared first, so a
// stale id reports BAD_EXPERT instead of reading a reused slot), and the
// compute stream waits for those copies.  The copies are spread over the
// pool's own copy streams, forked from the caller's copy stream and joined
// back into it, so several are in flight at once (a fill of one expert is
// three transfers of ~0.3 MB, where per-copy overhead is a large share).  Pinned
// slots are released when the caller says the work using them is done
// (redlite_moe_pool_complete) or when a CUDA event recorded after that work
// completes (redlite_moe_pool_release).
#include <new>
#include <vector>

#include "internal.cuh"

struct redlite_moe_pool {
  int n_experts = 0, capacity = 0;
  std::vector<int32_t> slot_expert;  // expert held by each slot, -1 if free
  std::vector<int32_t> expert_slot;  // slot of each expert, -1 if not resident
  std::vector<int64_t> last_use;     // recency tick of each slot
  std::vector<int32_t> pins;         // in-flight calls holding each slot
  int64_t tick = 0, next_token = 1;
  struct Pending {
    int64_t token;
    std::vector<int32_t> slots;
    cudaEvent_t event;  // nullptr until released with an event
  };
  std::vector<Pending> pending;
  // copy streams of this pool (created on the first fill) with the events
  // that fork them from, and join them back into, the caller's copy stream
  static constexpr int kStreams = 8;
  cudaStream_t streams[kStreams] = {};
  cudaEvent_t fork = nullptr, join[kStreams] = {};
  bool streams_ok = false;
};

namespace {

void unpin(redlite_moe_pool *p, size_t i) {
  for (int32_t s : p->pending[i].slots) --p->pins[s];
  if (p->pending[i].event) cudaEventDestroy(p->pending[i].event);
  p->pending.erase(p->pending.begin() + (long)i);
}

// Retire every pending call whose release event has completed.
void poll_events(redlite_moe_pool *p) {
  for (size_t i = 0; i < p->pending.size();) {
    cudaEvent_t e = p->pending[i].event;
    if (!e) {
      ++i;
    } else if (cudaEventQuery(e) == cudaSuccess) {
      unpin(p, i);
    } else {
      (void)cudaGetLastError();  // cudaErrorNotReady is not an error to keep
      ++i;
    }
  }
}

// Slot-table updates of one acquire, passed by value: entry id[i] of the
// table becomes d[i] (an empty entry for an eviction).  One launch replaces
// a small pageable host -> device copy per entry.
constexpr int kMaxUpdates = 64;
struct TableUpdates {
  int32_t n;
  int32_t id[kMaxUpdates];
  redlite_moe_expert d[kMaxUpdates];
};
static_assert(sizeof(TableUpdates) <= 4096, "kernel parameters");

__global__ void table_update_kernel(const TableUpdates u, redlite_moe_expert *table) {
  const int i = threadIdx.x;
  if (i < u.n) table[u.id[i]] = u.d[i];
}

}  // namespace

extern "C" {

redlite_moe_pool *redlite_moe_pool_create(int32_t n_experts, int32_t capacity) {
  if (n_experts <= 0 || capacity <= 0) return nullptr;
  redlite_moe_pool *p = new (std::nothrow) redlite_moe_pool;
  if (!p) return nullptr;
  p->n_experts = n_experts;
  p->capacity = capacity;
  p->slot_expert.assign((size_t)capacity, -1);
  p->expert_slot.assign((size_t)n_experts, -1);
  p->last_use.assign((size_t)capacity, 0);
  p->pins.assign((size_t)capacity, 0);
  return p;
}

void redlite_moe_pool_destroy(redlite_moe_pool *p) {
  if (!p) return;
  for (auto &q : p->pending)
    if (q.event) cudaEventDestroy(q.event);
  for (int i = 0; i < redlite_moe_pool::kStreams; ++i) {
    if (p->streams[i]) cudaStreamDestroy(p->streams[i]);
    if (p->join[i]) cudaEventDestroy(p->join[i]);
  }
  if (p->fork) cudaEventDestroy(p->fork);
  delete p;
}

int32_t redlite_moe_pool_slot_of(const redlite_moe_pool *p, int32_t expert) {
  if (!p || expert < 0 || expert >= p->n_experts) return -1;
  return p->expert_slot[(size_t)expert];
}

int32_t redlite_moe_pool_pins(const redlite_moe_pool *p, int32_t slot) {
  if (!p || slot < 0 || slot >= p->capacity) return -1;
  return p->pins[(size_t)slot];
}

int redlite_moe_pool_plan(redlite_moe_pool *p, const int32_t *ids, int32_t n, int32_t *slot_of, int32_t *evicted,
                          uint8_t *miss, int64_t *token) {
  if (!p || n < 0 || (n > 0 && (!ids || !slot_of || !evicted || !miss)) || !token) return REDLITE_EINVAL;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= p->n_experts) return REDLITE_EINVAL;
  // hard capacity: the distinct selected experts must fit at once
  std::vector<uint8_t> selected((size_t)p->n_experts, 0);
  int distinct = 0;
  for (int i = 0; i < n; ++i)
    if (!selected[(size_t)ids[i]]) selected[(size_t)ids[i]] = 1, ++distinct;
  if (distinct > p->capacity) return REDLITE_ENOMEM;
  poll_events(p);
  // pass 1: the resident selected experts are hits and are protected (the
  // whole selection, not only the ids before a miss, is protected while the
  // misses are filled)
  std::vector<uint8_t> prot((size_t)p->capacity, 0);
  for (int i = 0; i < n; ++i) {
    const int32_t s = p->expert_slot[(size_t)ids[i]];
    miss[i] = s < 0;
    if (s >= 0) prot[(size_t)s] = 1;
  }
  // pass 2 (planned first, committed only if every miss finds a slot): a
  // free slot (lowest index), else the least recently used slot that is
  // neither protected nor in flight
  std::vector<int32_t> victims;
  std::vector<uint8_t> taken((size_t)p->capacity, 0);
  for (int i = 0; i < n; ++i) {
    if (!miss[i]) continue;
    bool dup = false;  // a repeated miss id shares the first occurrence's slot
    for (int j = 0; j < i && !dup; ++j) dup = miss[j] && ids[j] == ids[i];
    if (dup) continue;
    int best = -1;
    for (int s = 0; s < p->capacity && best < 0; ++s)
      if (p->slot_expert[(size_t)s] < 0 && !taken[(size_t)s]) best = s;
    if (best < 0)
      for (int s = 0; s < p->capacity; ++s)
        if (!prot[(size_t)s] && !taken[(size_t)s] && p->pins[(size_t)s] == 0 &&
            (best < 0 || p->last_use[(size_t)s] < p->last_use[(size_t)best]))
          best = s;
    if (best < 0) return REDLITE_EAGAIN;  // every candidate slot is in flight
    taken[(size_t)best] = 1;
    victims.push_back(best);
  }
  // commit: hits are refreshed in selection order, then each miss takes its
  // slot (and is refreshed) in selection order
  for (int i = 0; i < n; ++i) {
    evicted[i] = -1;
    if (!miss[i]) {
      slot_of[i] = p->expert_slot[(size_t)ids[i]];
      p->last_use[(size_t)slot_of[i]] = ++p->tick;
    }
  }
  size_t v = 0;
  for (int i = 0; i < n; ++i) {
    if (!miss[i]) continue;
    const int32_t already = p->expert_slot[(size_t)ids[i]];
    if (already >= 0) {  // repeated miss id: filled by its first occurrence
      slot_of[i] = already;
      miss[i] = 0;
      continue;
    }
    const int32_t s = victims[v++];
    const int32_t old = p->slot_expert[(size_t)s];
    if (old >= 0) p->expert_slot[(size_t)old] = -1;
    evicted[i] = old;
    p->slot_expert[(size_t)s] = ids[i];
    p->expert_slot[(size_t)ids[i]] = s;
    p->last_use[(size_t)s] = ++p->tick;
    slot_of[i] = s;
  }
  // pin the selection for the call that uses it
  redlite_moe_pool::Pending q;
  q.token = p->next_token++;
  q.event = nullptr;
  for (int i = 0; i < n; ++i) {
    bool seen = false;
    for (int32_t s : q.slots) seen |= s == slot_of[i];
    if (!seen) q.slots.push_back(slot_of[i]);
  }
  for (int32_t s : q.slots) ++p->pins[(size_t)s];
  *token = q.token;
  p->pending.push_back(std::move(q));
  return REDLITE_OK;
}

int redlite_moe_pool_complete(redlite_moe_pool *p, int64_t token) {
  if (!p) return REDLITE_EINVAL;
  for (size_t i = 0; i < p->pending.size(); ++i)
    if (p->pending[i].token == token) {
      unpin(p, i);
      return REDLITE_OK;
    }
  return REDLITE_EINVAL;
}

int redlite_moe_pool_release(redlite_moe_pool *p, int64_t token, void *stream) {
  if (!p) return REDLITE_EINVAL;
  for (auto &q : p->pending)
    if (q.token == token && !q.event) {
      if (cudaEventCreateWithFlags(&q.event, cudaEventDisableTiming) != cudaSuccess) {
        q.event = nullptr;
        return REDLITE_ECUDA;
      }
      if (cudaEventRecord(q.event, (cudaStream_t)stream) != cudaSuccess) return REDLITE_ECUDA;
      return REDLITE_OK;
    }
  return REDLITE_EINVAL;
}

int redlite_moe_pool_acquire(redlite_moe_pool *p, const int32_t *ids, int32_t n, const redlite_moe_expert *host_experts,
                             int32_t hidden, void *slots_dev, size_t slot_bytes, redlite_moe_expert *table_dev,
                             void *copy_stream, void *compute_stream, redlite_moe_pool_counters *counters,
                             int64_t *token) {
  using namespace redlite;
  if (!p || !host_experts || !slots_dev || !table_dev || hidden <= 0 || !token) return REDLITE_EINVAL;
  if (((uintptr_t)slots_dev & 15) || (slot_bytes & 15)) return REDLITE_EINVAL;
  // every selected expert's matrices fit one slot
  for (int i = 0; i < n; ++i) {
    if (!ids || ids[i] < 0 || ids[i] >= p->n_experts) return REDLITE_EINVAL;
    const redlite_moe_expert &h = host_experts[ids[i]];
    if ((h.qtype != kQ2 && h.qtype != kQ1) || h.ffn <= 0 || !h.gate || !h.up || !h.down) return REDLITE_EINVAL;
    const size_t gb = matrix_bytes(h.qtype, h.ffn, hidden), db = matrix_bytes(h.qtype, hidden, h.ffn);
    if (!gb || !db) return REDLITE_EUNSUPPORTED;
    if (2 * ((gb + 15) & ~size_t(15)) + db > slot_bytes) return REDLITE_ENOMEM;
  }
  std::vector<int32_t> slot((size_t)n), ev((size_t)n);
  std::vector<uint8_t> miss((size_t)n);
  const int rc = redlite_moe_pool_plan(p, ids, n, slot.data(), ev.data(), miss.data(), token);
  if (rc != REDLITE_OK) return rc;
  cudaStream_t cs = (cudaStream_t)copy_stream;
  int64_t loads = 0, hits = 0, evictions = 0, bytes = 0;
  static const redlite_moe_expert kEmpty = {0, 0, nullptr, nullptr, nullptr};
  TableUpdates upd;
  upd.n = 0;
  // table entries are written after every fill has landed: evicted entries
  // cleared, loaded entries set (flushed early if the batch is full)
  auto flush = [&]() -> bool {
    if (!upd.n) return true;
    table_update_kernel<<<1, kMaxUpdates, 0, cs>>>(upd, table_dev);
    upd.n = 0;
    return cudaGetLastError() == cudaSuccess;
  };
  int n_miss = 0;
  for (int i = 0; i < n; ++i) n_miss += miss[i] != 0;
  constexpr int S = redlite_moe_pool::kStreams;
  if (n_miss > 1 && !p->streams_ok) {
    bool ok = cudaEventCreateWithFlags(&p->fork, cudaEventDisableTiming) == cudaSuccess;
    for (int j = 0; ok && j < S; ++j)
      ok = cudaStreamCreateWithFlags(&p->streams[j], cudaStreamNonBlocking) == cudaSuccess &&
           cudaEventCreateWithFlags(&p->join[j], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return REDLITE_ECUDA;
    p->streams_ok = true;
  }
  // with several fills: fork the pool's streams from the caller's copy stream
  const int n_used = n_miss > 1 ? (n_miss < S ? n_miss : S) : 0;
  if (n_used) {
    if (cudaEventRecord(p->fork, cs) != cudaSuccess) return REDLITE_ECUDA;
    for (int j = 0; j < n_used; ++j)
      if (cudaStreamWaitEvent(p->streams[j], p->fork, 0) != cudaSuccess) return REDLITE_ECUDA;
  }
  for (int i = 0; i < n; ++i) {
    if (!miss[i]) {
      ++hits;
      continue;
    }
    const cudaStream_t fs = n_used ? p->streams[loads % n_used] : cs;
    const redlite_moe_expert &h = host_experts[ids[i]];
    const size_t gb = matrix_bytes(h.qtype, h.ffn, hidden), db = matrix_bytes(h.qtype, hidden, h.ffn);
    const size_t ga = (gb + 15) & ~size_t(15);
    uint8_t *base = (uint8_t *)slots_dev + (size_t)slot[i] * slot_bytes;
    redlite_moe_expert d{h.qtype, h.ffn, base, base + ga, base + 2 * ga};
    if (ev[i] >= 0) {
      ++evictions;
      upd.id[upd.n] = ev[i], upd.d[upd.n] = kEmpty, ++upd.n;
    }
    if (cudaMemcpyAsync(base, h.gate, gb, cudaMemcpyHostToDevice, fs) != cudaSuccess ||
        cudaMemcpyAsync(base + ga, h.up, gb, cudaMemcpyHostToDevice, fs) != cudaSuccess ||
        cudaMemcpyAsync(base + 2 * ga, h.down, db, cudaMemcpyHostToDevice, fs) != cudaSuccess)
      return REDLITE_ECUDA;
    upd.id[upd.n] = ids[i], upd.d[upd.n] = d, ++upd.n;
    ++loads;
    bytes += (int64_t)(2 * gb + db);
    if (upd.n > kMaxUpdates - 2) {
      // a full batch: its entries' fills must land first
      for (int j = 0; j < n_used; ++j)
        if (cudaEventRecord(p->join[j], p->streams[j]) != cudaSuccess ||
            cudaStreamWaitEvent(cs, p->join[j], 0) != cudaSuccess)
          return REDLITE_ECUDA;
      if (!flush()) return REDLITE_ECUDA;
    }
  }
  // join the pool's streams back into the caller's copy stream, then write
  // the table entries
  for (int j = 0; j < n_used; ++j)
    if (cudaEventRecord(p->join[j], p->streams[j]) != cudaSuccess || cudaStreamWaitEvent(cs, p->join[j], 0) != cudaSuccess)
      return REDLITE_ECUDA;
  if (!flush()) return REDLITE_ECUDA;
  if (loads && copy_stream != compute_stream) {
    // the work enqueued next on the compute stream waits for the fills
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return REDLITE_ECUDA;
    const bool ok = cudaEventRecord(e, cs) == cudaSuccess &&
                    cudaStreamWaitEvent((cudaStream_t)compute_stream, e, 0) == cudaSuccess;
    cudaEventDestroy(e);
    if (!ok) return REDLITE_ECUDA;
  }
  if (counters) {
    counters->loads += loads;
    counters->hits += hits;
    counters->evictions += evictions;
    counters->copies += 3 * loads;
    counters->bytes += bytes;
  }
  return REDLITE_OK;
}

}  // extern "C"
