// Host prefix-hash index of cached attention-map states (MapFlow article,
// 163.com, section on the three system components: states are indexed by a
// prefix hash that covers the preceding context, and one sender state can
// serve several downstream models).
//
// Hash: two 64-bit FNV-1a chains over little-endian token bytes.  The
// state of block k is the hash of (state of block k-1, tokens of block k), so
// a block's key covers the whole prefix up to it.  Chain b feeds every token
// through a splitmix64 finaliser first and starts from another offset, so the
// two halves of the 128-bit key are independent in practice.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "../../include/mapflow.h"

namespace {

constexpr uint64_t kFnvPrime = 0x100000001b3ull;
constexpr uint64_t kOffsetA = 0xcbf29ce484222325ull;
constexpr uint64_t kOffsetB = 0x84222325cbf29ce4ull;

inline uint64_t fnv_bytes(uint64_t h, const void* p, size_t n) {
  const unsigned char* b = static_cast<const unsigned char*>(p);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= kFnvPrime;
  }
  return h;
}

inline uint64_t splitmix(uint64_t x) {
  x += 0x9e3779b97f4a7c15ull;
  x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
  x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}

struct Key {
  uint64_t a, b;
  int32_t layer;
  bool operator==(const Key& o) const { return a == o.a && b == o.b && layer == o.layer; }
};

struct KeyHash {
  size_t operator()(const Key& k) const {
    return size_t(k.a ^ (k.b * 0x9e3779b97f4a7c15ull) ^ (uint64_t(uint32_t(k.layer)) << 17));
  }
};

struct Entry {
  mf_csr_cache cache;
  int32_t seq;
  int64_t blocks;
};

struct Index {
  std::unordered_map<Key, Entry, KeyHash> map;
};

}  // namespace

extern "C" {

mf_status mf_prefix_hash(const int32_t* tokens, int64_t n, int32_t B, uint64_t seed,
                         uint64_t* out) {
  if ((n > 0 && !tokens) || !out || n < 0 || B < 1) return MF_ERR_INVALID_ARG;
  uint64_t ha = kOffsetA ^ seed;
  uint64_t hb = kOffsetB ^ splitmix(seed);
  int64_t nb = (n + B - 1) / B;
  for (int64_t k = 0; k < nb; ++k) {
    uint64_t sa = fnv_bytes(kOffsetA, &ha, sizeof(ha));
    uint64_t sb = fnv_bytes(kOffsetB, &hb, sizeof(hb));
    int64_t lo = k * B, hi = lo + B < n ? lo + B : n;
    for (int64_t t = lo; t < hi; ++t) {
      uint32_t tok = uint32_t(tokens[t]);
      sa = fnv_bytes(sa, &tok, sizeof(tok));
      uint64_t mixed = splitmix(uint64_t(tok) ^ (uint64_t(t - lo) << 32));
      sb = fnv_bytes(sb, &mixed, sizeof(mixed));
    }
    ha = sa;
    hb = sb;
    out[2 * k] = ha;
    out[2 * k + 1] = hb;
  }
  return MF_OK;
}

mf_status mf_index_create(void** index) {
  if (!index) return MF_ERR_INVALID_ARG;
  *index = new Index();
  return MF_OK;
}

void mf_index_destroy(void* index) { delete static_cast<Index*>(index); }

mf_status mf_index_insert(void* index, const uint64_t* hashes, int64_t nblocks,
                          int32_t sender_layer, int32_t seq, const mf_csr_cache* cache) {
  if (!index || !hashes || !cache || nblocks < 1 || seq < 0) return MF_ERR_INVALID_ARG;
  Index* ix = static_cast<Index*>(index);
  for (int64_t k = 0; k < nblocks; ++k) {
    Key key{hashes[2 * k], hashes[2 * k + 1], sender_layer};
    ix->map[key] = Entry{*cache, seq, k + 1};
  }
  return MF_OK;
}

mf_status mf_index_lookup(void* index, const uint64_t* hashes, int64_t nblocks,
                          int32_t sender_layer, mf_csr_cache* cache, int32_t* seq,
                          int64_t* matched_blocks) {
  if (!index || (!hashes && nblocks > 0) || !cache || !seq || !matched_blocks || nblocks < 0)
    return MF_ERR_INVALID_ARG;
  Index* ix = static_cast<Index*>(index);
  for (int64_t k = nblocks; k >= 1; --k) {
    Key key{hashes[2 * (k - 1)], hashes[2 * (k - 1) + 1], sender_layer};
    auto it = ix->map.find(key);
    if (it != ix->map.end() && it->second.blocks == k) {
      *cache = it->second.cache;
      *seq = it->second.seq;
      *matched_blocks = k;
      return MF_OK;
    }
  }
  return MF_ERR_NOT_FOUND;
}

int64_t mf_index_size(void* index) {
  return index ? int64_t(static_cast<Index*>(index)->map.size()) : 0;
}

}  // extern "C"
