// Expert slot manager: a host-side LRU over (layer, expert) keys whose values
// are slots of a caller-owned device pool.  It mirrors the engine's global
// LRU expert cache (FreeToken model guide, offload strategy: OffloadMoeCache
// with per-(layer, expert) recency and a guard that refuses a cache too small
// to make progress; sm89-moe-offload README, --moe-cache-size).
//
// acquire(layer, ids):
//   1. every requested expert that is resident is a hit: it moves to the
//      most-recently-used end and is pinned for this call;
//   2. every miss takes a free slot, else evicts the least recently used
//      slot not pinned by this call, and is filled from its pinned host bank
//      with one cudaMemcpyAsync on the copy stream.  A fill that reuses a
//      slot waits on the copy stream only for the compute work that last
//      used that slot: each acquire records an event on the compute stream
//      (everything enqueued so far), which becomes the last-use mark of the
//      slots the previous acquire handed out.  So fills for the next layer
//      overlap the current layer's kernels unless they evict its slots;
//   3. the device slot table [E] is uploaded on the copy stream, an event is
//      recorded there and the compute stream waits on it.
// More distinct experts than capacity -> FT_ERR_CAPACITY (nothing changes).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "ftmoe.h"

namespace ftmoe {
void set_last_error(const char* msg);
}

struct ft_slot_mgr {
  int capacity = 0;
  ft_nvfp4_slot_layout layout{};
  uint8_t* pool = nullptr;
  // LRU list of resident keys, most recent at the front
  std::list<uint64_t> lru;
  struct Entry {
    int slot;
    std::list<uint64_t>::iterator it;
  };
  std::unordered_map<uint64_t, Entry> resident;
  std::unordered_map<uint64_t, const void*> banks;
  std::vector<int> free_slots;
  std::vector<int32_t> host_table;      // staging copy of the last uploaded table
  // page-locked staging of the table uploads: a ring, so that an acquire
  // blocks the host only when the upload of kStage calls ago is still
  // pending (with one buffer, every acquire waited for the previous call's
  // fills, which left the copy engine idle while the host queued the next)
  static constexpr int kStage = 8;
  int32_t* pinned_table[kStage] = {};
  cudaEvent_t staged[kStage] = {};     // upload of pinned_table[i] (and the fills before it) done
  int pinned_table_len = 0;
  int next_stage = 0;
  // last-use marks: a ring of events recorded on the compute stream, one per
  // acquire; slot_mark[s] indexes the ring (-1: never used).  A ring entry may
  // be re-recorded later than the use it marks, which only makes a wait longer.
  static constexpr int kMarks = 64;
  cudaEvent_t marks[kMarks] = {};
  int next_mark = 0;
  std::vector<int> slot_mark;
  std::vector<int> prev_slots;          // slots handed out by the previous acquire
  ft_slot_stats_t stats{};
  int inject_failures = 0;
  bool host_only = false;               // FT_SLOT_HOST_ONLY: bookkeeping only, no CUDA calls
  std::mutex mu;
};

static inline uint64_t slot_key(int layer, int expert) {
  return (uint64_t(uint32_t(layer)) << 32) | uint32_t(expert);
}

extern "C" int ft_slot_create(ft_slot_mgr** mgr, int capacity, const ft_nvfp4_slot_layout* layout,
                              void* device_pool, int flags) {
  const bool host_only = (flags & FT_SLOT_HOST_ONLY) != 0;
  if (!mgr || !layout || (!device_pool && !host_only) || capacity <= 0 || capacity > layout->num_slots) {
    ftmoe::set_last_error("ft_slot_create: bad argument");
    return FT_ERR_INVALID_ARG;
  }
  auto* m = new ft_slot_mgr();
  m->capacity = capacity;
  m->layout = *layout;
  m->pool = static_cast<uint8_t*>(device_pool);
  m->host_only = host_only;
  for (int s = capacity - 1; s >= 0; --s) m->free_slots.push_back(s);
  m->slot_mark.assign(capacity, -1);
  bool ok = true;
  if (!host_only) {
    for (int i = 0; i < ft_slot_mgr::kStage && ok; ++i)
      ok = cudaEventCreateWithFlags(&m->staged[i], cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < ft_slot_mgr::kMarks && ok; ++i)
      ok = cudaEventCreateWithFlags(&m->marks[i], cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    ftmoe::set_last_error("ft_slot_create: cudaEventCreate failed");
    ft_slot_destroy(m);
    return FT_ERR_CUDA;
  }
  *mgr = m;
  return FT_OK;
}

extern "C" int ft_slot_register_host(ft_slot_mgr* m, int layer, int expert, const void* pinned_src) {
  if (!m || !pinned_src || layer < 0 || expert < 0) {
    ftmoe::set_last_error("ft_slot_register_host: bad argument");
    return FT_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> g(m->mu);
  m->banks[slot_key(layer, expert)] = pinned_src;
  return FT_OK;
}

extern "C" int ft_slot_inject_copy_failures(ft_slot_mgr* m, int count) {
  if (!m || count < 0) return FT_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(m->mu);
  m->inject_failures = count;
  return FT_OK;
}

extern "C" int ft_slot_acquire(ft_slot_mgr* m, int layer, const int32_t* ids, int n, int32_t* device_table,
                               int table_len, ft_stream_t compute, ft_stream_t copy) {
  if (!m || (n > 0 && !ids) || !device_table || table_len <= 0 || n < 0) {
    ftmoe::set_last_error("ft_slot_acquire: bad argument");
    return FT_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> g(m->mu);
  // distinct requested experts, in request order
  std::vector<int> want;
  want.reserve(n);
  {
    std::vector<char> seen(table_len, 0);
    for (int i = 0; i < n; ++i) {
      const int e = ids[i];
      if (e < 0 || e >= table_len) {
        ftmoe::set_last_error("ft_slot_acquire: expert id outside [0, table_len)");
        return FT_ERR_INVALID_ARG;
      }
      if (!seen[e]) { seen[e] = 1; want.push_back(e); }
    }
  }
  if ((int)want.size() > m->capacity) {
    ftmoe::set_last_error("ft_slot_acquire: more distinct experts than slots (cache too small)");
    return FT_ERR_CAPACITY;
  }
  for (int e : want) {
    const uint64_t key = slot_key(layer, e);
    if (!m->resident.count(key) && !m->banks.count(key)) {
      ftmoe::set_last_error("ft_slot_acquire: a missing expert has no registered host bank");
      return FT_ERR_NOT_RESIDENT;
    }
  }
  // the work enqueued on the compute stream so far is the last use of the
  // slots the previous acquire handed out
  if (!m->host_only && !m->prev_slots.empty()) {
    const int mk = m->next_mark;
    if (cudaEventRecord(m->marks[mk], reinterpret_cast<cudaStream_t>(compute)) != cudaSuccess) {
      ftmoe::set_last_error("ft_slot_acquire: recording the compute mark failed");
      return FT_ERR_CUDA;
    }
    m->next_mark = (mk + 1) % ft_slot_mgr::kMarks;
    for (int sl : m->prev_slots) m->slot_mark[sl] = mk;
    m->prev_slots.clear();
  }
  // pin: hits move to the front; they are protected from eviction by this call
  std::unordered_map<uint64_t, char> pinned;
  for (int e : want) {
    const uint64_t key = slot_key(layer, e);
    auto it = m->resident.find(key);
    pinned[key] = 1;
    if (it != m->resident.end()) {
      m->lru.splice(m->lru.begin(), m->lru, it->second.it);
      ++m->stats.hits;
    }
  }
  std::vector<int32_t> table(table_len, -1);
  const size_t slot_bytes = size_t(m->layout.slot_bytes);
  std::vector<char> waited(ft_slot_mgr::kMarks, 0);   // one stream wait per distinct mark
  struct Fill {
    int slot;
    uint64_t key;
    const uint8_t* src;
    bool fail;   // an injected failure (test hook)
  };
  std::vector<Fill> fills;
  // fills [from, end) did not happen: their slots are free again, their keys not resident
  auto rollback = [&](size_t from) {
    for (size_t r = from; r < fills.size(); ++r) {
      auto it = m->resident.find(fills[r].key);
      m->lru.erase(it->second.it);
      m->resident.erase(it);
      m->free_slots.push_back(fills[r].slot);
      --m->stats.misses;
      m->stats.bytes_h2d -= int64_t(slot_bytes);
    }
    fills.resize(from);
  };
  // hits first; the misses then take their slots in the order of their host
  // banks' addresses (stable: request order among equal addresses), so that
  // consecutive slots receive consecutive banks and the copies coalesce
  std::vector<int> misses;
  for (int e : want) {
    auto it = m->resident.find(slot_key(layer, e));
    if (it != m->resident.end()) table[e] = it->second.slot;
    else misses.push_back(e);
  }
  std::stable_sort(misses.begin(), misses.end(), [&](int a, int b) {
    return m->banks[slot_key(layer, a)] < m->banks[slot_key(layer, b)];
  });
  for (int e : misses) {
    const uint64_t key = slot_key(layer, e);
    int slot;
    if (!m->free_slots.empty()) {
      slot = m->free_slots.back();
      m->free_slots.pop_back();
    } else {
      // evict the least recently used entry that this call does not need
      auto victim = m->lru.end();
      for (auto r = m->lru.rbegin(); r != m->lru.rend(); ++r)
        if (!pinned.count(*r)) { victim = std::prev(r.base()); break; }
      if (victim == m->lru.end()) {
        rollback(0);
        ftmoe::set_last_error("ft_slot_acquire: no evictable slot");
        return FT_ERR_CAPACITY;
      }
      slot = m->resident[*victim].slot;
      m->resident.erase(*victim);
      m->lru.erase(victim);
      ++m->stats.evictions;
    }
    // the slot may still be read by compute work enqueued before: the fill
    // waits for the last use of this slot on the copy stream
    const int mk = m->slot_mark[slot];
    if (!m->host_only && mk >= 0 && !waited[mk]) {
      if (cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(copy), m->marks[mk], 0) != cudaSuccess) {
        m->free_slots.push_back(slot);
        rollback(0);
        ftmoe::set_last_error("ft_slot_acquire: ordering the fill after compute failed");
        return FT_ERR_CUDA;
      }
      waited[mk] = 1;
    }
    bool fail = false;
    if (m->inject_failures > 0) {
      --m->inject_failures;
      fail = true;
    }
    fills.push_back(Fill{slot, key, static_cast<const uint8_t*>(m->banks[key]), fail});
    m->lru.push_front(key);
    m->resident[key] = ft_slot_mgr::Entry{slot, m->lru.begin()};
    table[e] = slot;
    ++m->stats.misses;
    m->stats.bytes_h2d += int64_t(slot_bytes);
  }
  // The fills, one cudaMemcpyAsync per run of consecutive slots whose host
  // banks are consecutive too (banks registered in one page-locked block, and
  // slots freed in the order they were handed out, make long runs): each copy
  // has a fixed cost on the copy engine, so 128 fills of one layer become a
  // few large copies.  Every wait above is already enqueued before them.  A
  // failed copy leaves its run and every later one not resident.
  std::sort(fills.begin(), fills.end(), [](const Fill& a, const Fill& b) { return a.slot < b.slot; });
  for (size_t i = 0; i < fills.size();) {
    size_t j = i + 1;
    bool fail = fills[i].fail;
    while (j < fills.size() && fills[j].slot == fills[j - 1].slot + 1 &&
           fills[j].src == fills[j - 1].src + slot_bytes) {
      fail = fail || fills[j].fail;
      ++j;
    }
    cudaError_t err = fail ? cudaErrorUnknown : cudaSuccess;
    if (!fail && !m->host_only)
      err = cudaMemcpyAsync(m->pool + size_t(fills[i].slot) * slot_bytes, fills[i].src, (j - i) * slot_bytes,
                            cudaMemcpyHostToDevice, reinterpret_cast<cudaStream_t>(copy));
    if (err != cudaSuccess) {
      rollback(i);   // this run and the later ones hold nothing valid
      ftmoe::set_last_error("ft_slot_acquire: host-to-device fill failed");
      return FT_ERR_CUDA;
    }
    ++m->stats.copies;
    i = j;
  }
  m->host_table = table;
  for (int e : want) m->prev_slots.push_back(table[e]);
  if (m->host_only) {   // device_table is host memory in this mode
    std::memcpy(device_table, table.data(), size_t(table_len) * 4);
    return FT_OK;
  }
  // upload the table from page-locked staging so the copy stays asynchronous
  if (m->pinned_table_len < table_len) {
    // every pending upload must have finished reading the old buffers
    for (int i = 0; i < ft_slot_mgr::kStage; ++i) {
      cudaEventSynchronize(m->staged[i]);
      if (m->pinned_table[i]) cudaFreeHost(m->pinned_table[i]);
      m->pinned_table[i] = nullptr;
    }
    m->pinned_table_len = 0;
    for (int i = 0; i < ft_slot_mgr::kStage; ++i) {
      if (cudaMallocHost(reinterpret_cast<void**>(&m->pinned_table[i]), size_t(table_len) * 4) != cudaSuccess) {
        ftmoe::set_last_error("ft_slot_acquire: cudaMallocHost failed");
        return FT_ERR_CUDA;
      }
    }
    m->pinned_table_len = table_len;
  }
  const int st = m->next_stage;
  m->next_stage = (st + 1) % ft_slot_mgr::kStage;
  cudaEventSynchronize(m->staged[st]);   // the upload kStage calls ago finished reading this buffer
  std::memcpy(m->pinned_table[st], table.data(), size_t(table_len) * 4);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy);
  if (cudaMemcpyAsync(device_table, m->pinned_table[st], size_t(table_len) * 4, cudaMemcpyHostToDevice, cs) !=
          cudaSuccess ||
      cudaEventRecord(m->staged[st], cs) != cudaSuccess ||
      cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(compute), m->staged[st], 0) != cudaSuccess) {
    ftmoe::set_last_error("ft_slot_acquire: table upload failed");
    return FT_ERR_CUDA;
  }
  return FT_OK;
}

extern "C" int ft_slot_stats(const ft_slot_mgr* m, ft_slot_stats_t* out) {
  if (!m || !out) return FT_ERR_INVALID_ARG;
  *out = m->stats;
  return FT_OK;
}

extern "C" int ft_slot_destroy(ft_slot_mgr* m) {
  if (!m) return FT_ERR_INVALID_ARG;
  for (int i = 0; i < ft_slot_mgr::kStage; ++i) {
    if (m->staged[i]) {
      cudaEventSynchronize(m->staged[i]);
      cudaEventDestroy(m->staged[i]);
    }
    if (m->pinned_table[i]) cudaFreeHost(m->pinned_table[i]);
  }
  for (cudaEvent_t ev : m->marks)
    if (ev) cudaEventDestroy(ev);
  delete m;
  return FT_OK;
}
