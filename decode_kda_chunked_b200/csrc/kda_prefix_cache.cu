// Prefix cache over state snapshots (serving): the index and the pool copies.
//
// The serving layer keeps sparse state snapshots at 512-token block boundaries,
// and a request whose prompt starts with a cached prefix resumes from the state
// after it instead of running the whole prompt ("Kimi K3 开源日来了", Infra
// section, second layer).  A KDA state after a prefix depends only on the
// prefix, so one entry per block boundary is enough:
//
//   * kda_prefix_cache: a host index from the chained hash of a prompt's first j
//     blocks of token ids to a slot of a caller-owned device state pool.  The
//     hash of block j is FNV-1a (64-bit, Fowler-Noll-Vo) over the hash of block
//     j - 1 (0 before the first block) and the block's ids, each serialised
//     little-endian.  Every entry keeps its parent's hash and its block's ids
//     and a lookup compares both, so a hash collision cannot return the state of
//     another prompt.  With every slot taken, an insert evicts the least recently
//     used entry; a lookup or insert refreshes the blocks it walks deepest first,
//     so a chain's leading blocks are the last of it to go.
//   * kda_state_gather / kda_state_scatter: device copies between the pool and
//     dense per-request state arrays (the prefill's initial_state, its snapshots).
#include <cstring>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "kda_internal.cuh"

struct kda_prefix_cache {
  struct Entry {
    uint64_t parent;              // hash of the previous block (0 for the first)
    std::vector<int32_t> ids;     // the block's token ids
    int32_t slot;                 // pool slot holding the state after this block
    uint64_t stamp;               // call that last walked this entry
    std::list<uint64_t>::iterator lru;
  };
  int32_t block = 0, n_slots = 0;
  std::unordered_map<uint64_t, Entry> map;
  std::list<uint64_t> lru;        // most recently used first
  std::vector<int32_t> free_slots;
  uint64_t clock = 0;
  std::mutex mu;
};

namespace kda {
namespace {

constexpr uint64_t kFnvOffset = 14695981039346656037ull;
constexpr uint64_t kFnvPrime = 1099511628211ull;

uint64_t fnv_byte(uint64_t h, uint8_t b) { return (h ^ b) * kFnvPrime; }

uint64_t block_hash(uint64_t parent, const int32_t *ids, int32_t n) {
  uint64_t h = kFnvOffset;
  for (int s = 0; s < 64; s += 8) h = fnv_byte(h, (uint8_t)(parent >> s));
  for (int32_t i = 0; i < n; ++i) {
    const uint32_t u = (uint32_t)ids[i];
    for (int s = 0; s < 32; s += 8) h = fnv_byte(h, (uint8_t)(u >> s));
  }
  return h;
}

using Cache = kda_prefix_cache;

// The entry for block ids[0..block) under `parent`, or nullptr.
Cache::Entry *find(Cache *c, uint64_t key, uint64_t parent, const int32_t *ids) {
  auto it = c->map.find(key);
  if (it == c->map.end()) return nullptr;
  Cache::Entry &e = it->second;
  if (e.parent != parent || std::memcmp(e.ids.data(), ids, sizeof(int32_t) * c->block) != 0)
    return nullptr;
  return &e;
}

// Move the walked chain to the front of the LRU list, deepest block first, so
// its first block ends up the most recently used.
void refresh(Cache *c, const std::vector<uint64_t> &chain, uint64_t stamp) {
  for (auto k = chain.rbegin(); k != chain.rend(); ++k) {
    Cache::Entry &e = c->map.at(*k);
    c->lru.erase(e.lru);
    c->lru.push_front(*k);
    e.lru = c->lru.begin();
    e.stamp = stamp;
  }
}

constexpr int kCopyThreads = 256;

// dst[i] = pool[slots[i]] (zeros for slots[i] < 0); one grid row per state.
__global__ void gather_kernel(const float4 *pool, int n_slots, const int32_t *slots, size_t per,
                              float4 *dst, unsigned int *status) {
  const int i = blockIdx.y;
  const int s = slots[i];
  if (s >= n_slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, STATUS_BAD_SEQLENS);
    return;
  }
  float4 *d = dst + (size_t)i * per;
  const float4 *src = s >= 0 ? pool + (size_t)s * per : nullptr;
  for (size_t e = (size_t)blockIdx.x * kCopyThreads + threadIdx.x; e < per;
       e += (size_t)gridDim.x * kCopyThreads)
    d[e] = src ? src[e] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// pool[slots[i]] = src[i] for slots[i] >= 0.
__global__ void scatter_kernel(const float4 *src, const int32_t *slots, size_t per, float4 *pool,
                               int n_slots, unsigned int *status) {
  const int i = blockIdx.y;
  const int s = slots[i];
  if (s < 0) return;
  if (s >= n_slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, STATUS_BAD_SEQLENS);
    return;
  }
  const float4 *from = src + (size_t)i * per;
  float4 *to = pool + (size_t)s * per;
  for (size_t e = (size_t)blockIdx.x * kCopyThreads + threadIdx.x; e < per;
       e += (size_t)gridDim.x * kCopyThreads)
    to[e] = from[e];
}

bool copy_args_ok(const void *a, const void *b, const int32_t *slots, int32_t n, int32_t H,
                  int32_t dk, int32_t dv, int32_t n_slots) {
  if (n < 0 || H <= 0 || dk <= 0 || dv <= 0 || n_slots < 0) return false;
  if ((((size_t)dk * dv) & 3u) != 0) return false;
  if (n == 0) return true;
  if (!a || !b || !slots) return false;
  for (const void *p : {a, b, (const void *)slots})
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return false;
  return true;
}

dim3 copy_grid(size_t per, int32_t n) {
  size_t bx = (per + kCopyThreads * 4 - 1) / (kCopyThreads * 4);  // 4 float4 per thread
  if (bx < 1) bx = 1;
  if (bx > 1024) bx = 1024;
  return dim3((unsigned)bx, (unsigned)n);
}

}  // namespace
}  // namespace kda

extern "C" {

kda_prefix_cache *kda_prefix_cache_create(int32_t block_tokens, int32_t n_slots) {
  if (block_tokens <= 0 || n_slots <= 0) return nullptr;
  kda_prefix_cache *c = new (std::nothrow) kda_prefix_cache();
  if (!c) return nullptr;
  c->block = block_tokens;
  c->n_slots = n_slots;
  c->free_slots.reserve(n_slots);
  for (int32_t s = n_slots - 1; s >= 0; --s) c->free_slots.push_back(s);  // slot 0 first
  return c;
}

void kda_prefix_cache_destroy(kda_prefix_cache *c) { delete c; }

int32_t kda_prefix_cache_lookup(kda_prefix_cache *c, const int32_t *tokens, int32_t n_tokens,
                                int32_t max_tokens, int32_t *slot) {
  if (!c || !slot || n_tokens < 0 || (n_tokens > 0 && !tokens)) return -1;
  std::lock_guard<std::mutex> lock(c->mu);
  *slot = -1;
  const int32_t limit = max_tokens < n_tokens ? max_tokens : n_tokens;
  std::vector<uint64_t> chain;
  uint64_t parent = 0;
  for (int64_t end = c->block; end <= limit; end += c->block) {
    const int32_t *ids = tokens + (end - c->block);
    const uint64_t key = kda::block_hash(parent, ids, c->block);
    kda_prefix_cache::Entry *e = kda::find(c, key, parent, ids);
    if (!e) break;
    *slot = e->slot;
    chain.push_back(key);
    parent = key;
  }
  kda::refresh(c, chain, ++c->clock);
  return (int32_t)chain.size() * c->block;
}

int32_t kda_prefix_cache_insert(kda_prefix_cache *c, const int32_t *tokens, int32_t n_tokens,
                                int32_t first_block, int32_t *slots_out) {
  if (!c || n_tokens < 0 || first_block < 0 || (n_tokens > 0 && !tokens)) return -1;
  const int32_t nb = n_tokens / c->block;
  if (nb > 0 && !slots_out) return -1;
  std::lock_guard<std::mutex> lock(c->mu);
  const uint64_t stamp = ++c->clock;
  for (int32_t j = 0; j < nb; ++j) slots_out[j] = -1;
  std::vector<uint64_t> chain;
  uint64_t parent = 0;
  int32_t j = 0;
  for (; j < nb; ++j) {
    const int32_t *ids = tokens + (size_t)j * c->block;
    const uint64_t key = kda::block_hash(parent, ids, c->block);
    if (kda_prefix_cache::Entry *e = kda::find(c, key, parent, ids)) {
      // cached already (its state is the same): marked and moved to the front now, so
      // the evictions below never take a block of this prompt while others remain
      e->stamp = stamp;
      c->lru.erase(e->lru);
      c->lru.push_front(key);
      e->lru = c->lru.begin();
      chain.push_back(key);
      parent = key;
      continue;
    }
    if (j < first_block) break;  // a block whose state the caller cannot supply
    int32_t slot = -1;
    auto clash = c->map.find(key);
    if (clash != c->map.end()) {  // same hash, another block: take over its slot
      slot = clash->second.slot;
      c->lru.erase(clash->second.lru);
      c->map.erase(clash);
    } else if (!c->free_slots.empty()) {
      slot = c->free_slots.back();
      c->free_slots.pop_back();
    } else {
      // evict the least recently used entry, unless this call walked it
      const uint64_t victim = c->lru.back();
      auto v = c->map.find(victim);
      if (v->second.stamp == stamp) break;
      slot = v->second.slot;
      c->lru.pop_back();
      c->map.erase(v);
    }
    kda_prefix_cache::Entry e;
    e.parent = parent;
    e.ids.assign(ids, ids + c->block);
    e.slot = slot;
    e.stamp = stamp;
    c->lru.push_front(key);
    e.lru = c->lru.begin();
    c->map.emplace(key, std::move(e));
    slots_out[j] = slot;
    chain.push_back(key);
    parent = key;
  }
  kda::refresh(c, chain, stamp);
  return j;
}

int32_t kda_prefix_cache_size(const kda_prefix_cache *c) {
  if (!c) return -1;
  std::lock_guard<std::mutex> lock(const_cast<kda_prefix_cache *>(c)->mu);
  return (int32_t)c->map.size();
}

kda_status kda_state_gather(const float *pool, int32_t n_slots, const int32_t *slots, int32_t n,
                            int32_t H, int32_t dk, int32_t dv, float *dst, void *stream) {
  using namespace kda;
  if (!copy_args_ok(pool, dst, slots, n, H, dk, dv, n_slots)) return KDA_ERR_INVALID_ARG;
  if (n == 0) return KDA_OK;
  const size_t per = (size_t)H * dk * dv / 4;
  const char *plo = reinterpret_cast<const char *>(pool), *dlo = reinterpret_cast<const char *>(dst);
  if (dlo < plo + (size_t)n_slots * per * 16 && plo < dlo + (size_t)n * per * 16)
    return KDA_ERR_INVALID_ARG;  // the pool and dst overlap
  unsigned int *status = device_status_word();
  if (!status) return KDA_ERR_CUDA;
  gather_kernel<<<copy_grid(per, n), kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4 *>(pool), n_slots, slots, per, reinterpret_cast<float4 *>(dst),
      status);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_state_scatter(const float *src, const int32_t *slots, int32_t n, int32_t H,
                             int32_t dk, int32_t dv, float *pool, int32_t n_slots, void *stream) {
  using namespace kda;
  if (!copy_args_ok(src, pool, slots, n, H, dk, dv, n_slots)) return KDA_ERR_INVALID_ARG;
  if (n == 0) return KDA_OK;
  const size_t per = (size_t)H * dk * dv / 4;
  const char *plo = reinterpret_cast<const char *>(pool), *slo = reinterpret_cast<const char *>(src);
  if (slo < plo + (size_t)n_slots * per * 16 && plo < slo + (size_t)n * per * 16)
    return KDA_ERR_INVALID_ARG;  // the pool and src overlap
  unsigned int *status = device_status_word();
  if (!status) return KDA_ERR_CUDA;
  scatter_kernel<<<copy_grid(per, n), kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4 *>(src), slots, per, reinterpret_cast<float4 *>(pool), n_slots,
      status);
  return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
