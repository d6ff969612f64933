// tier.cu -- L1 <-> L2 page tiering for the Hierarchical KV Cache (WorldAttention
// §3.2, "Hierarchical KV Cache": pages that are not active leave GPU memory for CPU
// DRAM under an LRU policy and come back on demand; a side stream prefetches pages
// that are predicted to be needed).
//
// A tier owns no memory: the caller gives a device pool of n_slots page slots (the
// L1 tier, K and V) and pinned host memory holding every page (the L2 tier).  The
// tier keeps the page -> slot map, the LRU order and dirty bits, and issues the
// copies: on the caller's stream for demand misses (ordered with the kernels that
// use the slots), on its own stream for prefetches (ordered by events).  With no
// buffers at all it only keeps the books, which is how the replacement policy is
// tested without a GPU.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "wa_internal.h"

struct wa_tier {
  int n_pages = 0, n_slots = 0;
  size_t page_bytes = 0;
  char* host_k = nullptr;
  char* host_v = nullptr;
  char* slot_k = nullptr;
  char* slot_v = nullptr;
  bool copies = false;                 // false: bookkeeping only
  std::vector<int> slot_of;            // page -> slot, -1 when not resident
  std::vector<int> page_in;            // slot -> page, -1 when free
  std::vector<unsigned long long> last_use;   // slot -> LRU clock of its last hand-out
  std::vector<char> dirty;             // slot written on the device since it was loaded
  std::vector<char> prefetching;       // slot filled by a prefetch the caller has not waited on
  std::vector<cudaEvent_t> filled;     // slot -> recorded after its prefetch copy
  std::vector<char> host_pending;      // page -> a write-back of it may still be in flight
  std::vector<cudaEvent_t> host_done;  // page -> recorded after its write-back
  cudaEvent_t released = nullptr;      // the caller's stream after the last wa_tier_release
  unsigned long long clock = 0, released_clock = 0;
  bool any_release = false;
  cudaStream_t side = nullptr;
  wa_tier_stats stats{};
  std::mutex mu;
};

namespace {

using wa::set_error;

wa_status cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return WA_OK;
  return set_error(WA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Copy page `page` between host and slot `slot` (both K and V) on `st`.
wa_status copy_page(wa_tier* t, int page, int slot, bool to_device, cudaStream_t st) {
  const size_t hp = static_cast<size_t>(page) * t->page_bytes;
  const size_t sp = static_cast<size_t>(slot) * t->page_bytes;
  const cudaMemcpyKind kind = to_device ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
  for (int kv = 0; kv < 2; ++kv) {
    char* h = (kv ? t->host_v : t->host_k) + hp;
    char* s = (kv ? t->slot_v : t->slot_k) + sp;
    const cudaError_t e = to_device ? cudaMemcpyAsync(s, h, t->page_bytes, kind, st)
                                    : cudaMemcpyAsync(h, s, t->page_bytes, kind, st);
    if (e != cudaSuccess) return cuda_ok(e, "page copy");
  }
  if (to_device) t->stats.bytes_h2d += 2 * static_cast<long long>(t->page_bytes);
  else t->stats.bytes_d2h += 2 * static_cast<long long>(t->page_bytes);
  return WA_OK;
}

// Free slot first, else the least recently handed-out slot that is not `taken` and,
// for a prefetch (`released_only`), was handed out no later than the last release
// and does not hold a prefetched page nobody has asked for yet.
int pick_victim(const wa_tier* t, const std::vector<char>& taken, bool released_only) {
  int best = -1;
  for (int s = 0; s < t->n_slots; ++s) {
    if (taken[s]) continue;
    if (t->page_in[s] < 0) return s;
    if (released_only &&
        (!t->any_release || t->last_use[s] > t->released_clock || t->prefetching[s]))
      continue;
    if (best < 0 || t->last_use[s] < t->last_use[best]) best = s;
  }
  return best;
}

// Empty slot `s` (writing its page back if dirty) and load `page` into it, on `st`.
wa_status fill_slot(wa_tier* t, int s, int page, cudaStream_t st) {
  const int old = t->page_in[s];
  if (old >= 0) {
    ++t->stats.evictions;
    if (t->dirty[s]) {
      ++t->stats.writebacks;
      if (t->copies) {
        wa_status e = copy_page(t, old, s, false, st);
        if (e != WA_OK) return e;
        e = cuda_ok(cudaEventRecord(t->host_done[old], st), "event record");
        if (e != WA_OK) return e;
        t->host_pending[old] = 1;
      }
    }
    t->slot_of[old] = -1;
  }
  if (t->copies) {
    if (t->host_pending[page]) {   // the host copy is current only once its write-back lands
      wa_status e = cuda_ok(cudaStreamWaitEvent(st, t->host_done[page], 0), "stream wait");
      if (e != WA_OK) return e;
    }
    wa_status e = copy_page(t, page, s, true, st);
    if (e != WA_OK) return e;
  }
  t->page_in[s] = page;
  t->slot_of[page] = s;
  t->dirty[s] = 0;
  t->prefetching[s] = 0;
  return WA_OK;
}

wa_status check_pages(const wa_tier* t, const int32_t* pages, int n) {
  if (n < 0 || (n > 0 && !pages)) return set_error(WA_ERR_INVALID_ARG, "bad page list");
  for (int i = 0; i < n; ++i)
    if (pages[i] < 0 || pages[i] >= t->n_pages)
      return set_error(WA_ERR_INVALID_ARG, "page id %d out of range [0, %d)", pages[i], t->n_pages);
  return WA_OK;
}

}  // namespace

extern "C" {

wa_status wa_tier_create(int n_pages, int n_slots, size_t page_bytes, void* host_k, void* host_v,
                         void* slot_k, void* slot_v, wa_tier** out) {
  if (!out) return set_error(WA_ERR_INVALID_ARG, "NULL output");
  *out = nullptr;
  if (n_pages < 1 || n_slots < 1 || page_bytes == 0)
    return set_error(WA_ERR_INVALID_ARG, "need n_pages >= 1, n_slots >= 1, page_bytes > 0");
  const bool any = host_k || host_v || slot_k || slot_v;
  const bool all = host_k && host_v && slot_k && slot_v;
  if (any && !all) return set_error(WA_ERR_INVALID_ARG, "give all four buffers or none");
  wa_tier* t = new wa_tier;
  t->n_pages = n_pages;
  t->n_slots = n_slots;
  t->page_bytes = page_bytes;
  t->host_k = static_cast<char*>(host_k);
  t->host_v = static_cast<char*>(host_v);
  t->slot_k = static_cast<char*>(slot_k);
  t->slot_v = static_cast<char*>(slot_v);
  t->copies = all;
  t->slot_of.assign(n_pages, -1);
  t->page_in.assign(n_slots, -1);
  t->last_use.assign(n_slots, 0);
  t->dirty.assign(n_slots, 0);
  t->prefetching.assign(n_slots, 0);
  t->host_pending.assign(n_pages, 0);
  if (all) {
    bool ok = cudaStreamCreateWithFlags(&t->side, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&t->released, cudaEventDisableTiming) == cudaSuccess;
    t->filled.assign(n_slots, nullptr);
    t->host_done.assign(n_pages, nullptr);
    for (int s = 0; ok && s < n_slots; ++s)
      ok = cudaEventCreateWithFlags(&t->filled[s], cudaEventDisableTiming) == cudaSuccess;
    for (int p = 0; ok && p < n_pages; ++p)
      ok = cudaEventCreateWithFlags(&t->host_done[p], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      wa_tier_destroy(t);
      return set_error(WA_ERR_CUDA, "could not create the tier's stream and events");
    }
  }
  *out = t;
  return WA_OK;
}

wa_status wa_tier_destroy(wa_tier* t) {
  if (!t) return WA_OK;
  if (t->side) cudaStreamSynchronize(t->side);
  for (cudaEvent_t e : t->filled) if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : t->host_done) if (e) cudaEventDestroy(e);
  if (t->released) cudaEventDestroy(t->released);
  if (t->side) cudaStreamDestroy(t->side);
  delete t;
  return WA_OK;
}

wa_status wa_tier_ensure(wa_tier* t, const int32_t* pages, int n, int32_t* slots_out, void* stream) {
  if (!t || !slots_out) return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lock(t->mu);
  wa_status e = check_pages(t, pages, n);
  if (e != WA_OK) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // slots of this request are never chosen as victims within it
  std::vector<char> taken(t->n_slots, 0);
  int distinct = 0;
  for (int i = 0; i < n; ++i) {
    bool seen = false;
    for (int k = 0; k < i; ++k) seen |= pages[k] == pages[i];
    if (seen) continue;
    ++distinct;
    if (t->slot_of[pages[i]] >= 0) taken[t->slot_of[pages[i]]] = 1;
  }
  if (distinct > t->n_slots)
    return set_error(WA_ERR_INVALID_ARG, "%d distinct pages requested, %d slots", distinct, t->n_slots);
  for (int i = 0; i < n; ++i) {
    const int p = pages[i];
    int s = t->slot_of[p];
    if (s >= 0) {
      if (t->prefetching[s]) {
        ++t->stats.prefetch_hits;
        if (t->copies) {
          e = cuda_ok(cudaStreamWaitEvent(st, t->filled[s], 0), "stream wait");
          if (e != WA_OK) return e;
        }
        t->prefetching[s] = 0;
      } else {
        ++t->stats.hits;
      }
    } else {
      ++t->stats.misses;
      s = pick_victim(t, taken, false);
      if (t->copies && t->prefetching[s]) {   // a victim still being prefetched
        e = cuda_ok(cudaStreamWaitEvent(st, t->filled[s], 0), "stream wait");
        if (e != WA_OK) return e;
      }
      e = fill_slot(t, s, p, st);
      if (e != WA_OK) return e;
      taken[s] = 1;
    }
    t->last_use[s] = ++t->clock;
    slots_out[i] = s;
  }
  return WA_OK;
}

wa_status wa_tier_release(wa_tier* t, void* stream) {
  if (!t) return set_error(WA_ERR_INVALID_ARG, "NULL tier");
  std::lock_guard<std::mutex> lock(t->mu);
  if (t->copies) {
    wa_status e = cuda_ok(cudaEventRecord(t->released, static_cast<cudaStream_t>(stream)), "event record");
    if (e != WA_OK) return e;
  }
  t->released_clock = t->clock;
  t->any_release = true;
  return WA_OK;
}

wa_status wa_tier_prefetch(wa_tier* t, const int32_t* pages, int n, int* issued) {
  if (!t) return set_error(WA_ERR_INVALID_ARG, "NULL tier");
  std::lock_guard<std::mutex> lock(t->mu);
  wa_status e = check_pages(t, pages, n);
  if (e != WA_OK) return e;
  std::vector<char> taken(t->n_slots, 0);
  for (int i = 0; i < n; ++i)
    if (t->slot_of[pages[i]] >= 0) taken[t->slot_of[pages[i]]] = 1;
  int count = 0;
  bool waited = false;
  for (int i = 0; i < n; ++i) {
    const int p = pages[i];
    if (t->slot_of[p] >= 0) continue;
    const int s = pick_victim(t, taken, true);
    if (s < 0) break;                      // a hint: nothing evictable right now
    if (t->copies && t->page_in[s] >= 0 && !waited) {
      // the slot's last readers were enqueued on the caller's stream before the release
      e = cuda_ok(cudaStreamWaitEvent(t->side, t->released, 0), "stream wait");
      if (e != WA_OK) return e;
      waited = true;
    }
    e = fill_slot(t, s, p, t->side);
    if (e != WA_OK) return e;
    if (t->copies) {
      e = cuda_ok(cudaEventRecord(t->filled[s], t->side), "event record");
      if (e != WA_OK) return e;
    }
    t->prefetching[s] = 1;
    t->last_use[s] = ++t->clock;
    taken[s] = 1;
    ++count;
  }
  t->stats.prefetches += count;
  if (issued) *issued = count;
  return WA_OK;
}

wa_status wa_tier_mark_dirty(wa_tier* t, int32_t page) {
  if (!t) return set_error(WA_ERR_INVALID_ARG, "NULL tier");
  std::lock_guard<std::mutex> lock(t->mu);
  if (page < 0 || page >= t->n_pages || t->slot_of[page] < 0)
    return set_error(WA_ERR_INVALID_ARG, "page %d is not resident", page);
  t->dirty[t->slot_of[page]] = 1;
  return WA_OK;
}

wa_status wa_tier_flush(wa_tier* t, void* stream) {
  if (!t) return set_error(WA_ERR_INVALID_ARG, "NULL tier");
  std::lock_guard<std::mutex> lock(t->mu);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int s = 0; s < t->n_slots; ++s) {
    const int p = t->page_in[s];
    if (p < 0 || !t->dirty[s]) continue;
    ++t->stats.writebacks;
    if (t->copies) {
      if (t->prefetching[s]) {
        wa_status e = cuda_ok(cudaStreamWaitEvent(st, t->filled[s], 0), "stream wait");
        if (e != WA_OK) return e;
      }
      wa_status e = copy_page(t, p, s, false, st);
      if (e != WA_OK) return e;
      e = cuda_ok(cudaEventRecord(t->host_done[p], st), "event record");
      if (e != WA_OK) return e;
      t->host_pending[p] = 1;
    }
    t->dirty[s] = 0;
  }
  return WA_OK;
}

wa_status wa_tier_slot_of(wa_tier* t, int32_t page, int32_t* slot) {
  if (!t || !slot) return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lock(t->mu);
  if (page < 0 || page >= t->n_pages) return set_error(WA_ERR_INVALID_ARG, "page out of range");
  *slot = t->slot_of[page];
  return WA_OK;
}

wa_status wa_tier_get_stats(wa_tier* t, wa_tier_stats* out) {
  if (!t || !out) return set_error(WA_ERR_INVALID_ARG, "NULL pointer");
  std::lock_guard<std::mutex> lock(t->mu);
  *out = t->stats;
  return WA_OK;
}

}  // extern "C"
