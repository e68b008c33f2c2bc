// prefix_cache.cpp -- host side of prefix caching: chained per-block hashes of a
// request's tokens and a hash -> physical block map with the longest-hit lookup.
//
// The scheduler hashes every request in 16-token blocks and looks the hashes up,
// in order, in the map from block hash to cached block; every hit reuses that
// block's KV as it is (shengyayun.com 关键实现细节 item 2; hn.213312.xyz section
// 二, item 2).  Only full blocks are hashed: a trailing partial block is never
// reused (shengyayun.com 关键实现细节 item 1, last sentence).  A block's hash
// covers its parent's hash as well as its own tokens, so equal hashes mean equal
// whole prefixes and the walk can stop at the first miss.
//
// Hashes: FNV-1a 64 (fast, the default) or SHA-256 (FIPS 180-4, for callers who
// want collision resistance).  Both digest the same byte string per block:
//   parent digest (32 bytes) || the block's 16 token ids as little-endian int32.
// The first block's parent is the caller's root digest (zeros by default; a
// caller may fold extra keys such as an adapter id into it).
// An FNV-1a digest is its 64-bit value little-endian in bytes 0..7, zeros after.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <unordered_map>

#include "../../include/pa.h"

namespace {

constexpr int kBlockTokens = 16;
constexpr int kDigest = 32;

// ---------------------------------------------------------------- FNV-1a 64
uint64_t fnv1a64(const uint8_t *p, size_t n)
{
    uint64_t h = 14695981039346656037ull; // offset basis
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull; // 2^40 + 2^8 + 0xb3
    }
    return h;
}

// ---------------------------------------------------------------- SHA-256
// The round constants and initial hash value are derived at first use from
// their definition (FIPS 180-4 section 4.2.2 and 5.3.3): the first 32 bits of
// the fractional parts of the cube roots of the first 64 primes, and of the
// square roots of the first 8 primes.  Exact integer roots on 128-bit values.
struct Sha256Consts {
    uint32_t k[64];
    uint32_t h0[8];
};

unsigned __int128 iroot(unsigned __int128 x, int e) // floor(x^(1/e)), e = 2 or 3
{
    unsigned __int128 lo = 0, hi = (unsigned __int128)1 << (e == 2 ? 40 : 36); // roots here are < 2^35
    while (lo < hi) {
        const unsigned __int128 mid = lo + (hi - lo + 1) / 2;
        unsigned __int128 p = mid * mid;
        bool le;
        if (e == 2) {
            le = p <= x;
        } else {
            le = p <= x / mid && p * mid <= x;
        }
        if (le)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

const Sha256Consts &sha256_consts()
{
    static Sha256Consts c;
    static std::once_flag once;
    std::call_once(once, [] {
        int primes[64], n = 0;
        for (int v = 2; n < 64; ++v) {
            bool prime = true;
            for (int d = 2; d * d <= v; ++d)
                if (v % d == 0) {
                    prime = false;
                    break;
                }
            if (prime)
                primes[n++] = v;
        }
        for (int i = 0; i < 64; ++i) // frac(cbrt(p)) * 2^32 = floor(cbrt(p * 2^96)) mod 2^32
            c.k[i] = (uint32_t)iroot((unsigned __int128)primes[i] << 96, 3);
        for (int i = 0; i < 8; ++i) // frac(sqrt(p)) * 2^32 = floor(sqrt(p * 2^64)) mod 2^32
            c.h0[i] = (uint32_t)iroot((unsigned __int128)primes[i] << 64, 2);
    });
    return c;
}

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void sha256(const uint8_t *msg, size_t n, uint8_t out[32])
{
    const Sha256Consts &c = sha256_consts();
    uint32_t h[8];
    std::memcpy(h, c.h0, sizeof h);
    // padding: 0x80, zeros, 64-bit big-endian bit length, to a multiple of 64 bytes
    const size_t total = ((n + 9 + 63) / 64) * 64;
    uint8_t buf[128];
    for (size_t off = 0; off < total; off += 64) {
        const uint8_t *blk;
        if (off + 64 <= n) {
            blk = msg + off;
        } else {
            for (size_t i = 0; i < 64; ++i) {
                const size_t j = off + i;
                uint8_t b = 0;
                if (j < n)
                    b = msg[j];
                else if (j == n)
                    b = 0x80;
                else if (j >= total - 8)
                    b = (uint8_t)(((uint64_t)n * 8) >> (8 * (total - 1 - j)));
                buf[i] = b;
            }
            blk = buf;
        }
        uint32_t w[64];
        for (int t = 0; t < 16; ++t)
            w[t] = (uint32_t)blk[4 * t] << 24 | (uint32_t)blk[4 * t + 1] << 16 | (uint32_t)blk[4 * t + 2] << 8 |
                   (uint32_t)blk[4 * t + 3];
        for (int t = 16; t < 64; ++t) {
            const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
            const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
            w[t] = w[t - 16] + s0 + w[t - 7] + s1;
        }
        uint32_t a = h[0], b = h[1], cc = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
        for (int t = 0; t < 64; ++t) {
            const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
            const uint32_t ch = (e & f) ^ (~e & g);
            const uint32_t t1 = hh + S1 + ch + c.k[t] + w[t];
            const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
            const uint32_t maj = (a & b) ^ (a & cc) ^ (b & cc);
            const uint32_t t2 = S0 + maj;
            hh = g;
            g = f;
            f = e;
            e = d + t1;
            d = cc;
            cc = b;
            b = a;
            a = t1 + t2;
        }
        h[0] += a;
        h[1] += b;
        h[2] += cc;
        h[3] += d;
        h[4] += e;
        h[5] += f;
        h[6] += g;
        h[7] += hh;
    }
    for (int i = 0; i < 8; ++i)
        for (int j = 0; j < 4; ++j)
            out[4 * i + j] = (uint8_t)(h[i] >> (24 - 8 * j));
}

// ---------------------------------------------------------------- block digest
void block_digest(const uint8_t parent[kDigest], const int32_t *tokens, int32_t algo, uint8_t out[kDigest])
{
    uint8_t msg[kDigest + 4 * kBlockTokens];
    std::memcpy(msg, parent, kDigest);
    for (int i = 0; i < kBlockTokens; ++i) {
        const uint32_t t = (uint32_t)tokens[i];
        for (int b = 0; b < 4; ++b)
            msg[kDigest + 4 * i + b] = (uint8_t)(t >> (8 * b));
    }
    if (algo == PA_HASH_SHA256) {
        sha256(msg, sizeof msg, out);
    } else {
        const uint64_t h = fnv1a64(msg, sizeof msg);
        std::memset(out, 0, kDigest);
        for (int b = 0; b < 8; ++b)
            out[b] = (uint8_t)(h >> (8 * b));
    }
}

struct DigestHash {
    size_t operator()(const std::string &s) const
    {
        uint64_t v;
        std::memcpy(&v, s.data(), sizeof v); // digests are already well mixed
        return (size_t)v;
    }
};

} // namespace

struct pa_prefix_cache {
    std::mutex mu;
    std::unordered_map<std::string, int32_t, DigestHash> by_hash; // block hash -> physical block
    std::unordered_map<int32_t, std::string> by_block;            // physical block -> its hash
};

extern "C" {

pa_status_t pa_prefix_block_hashes(const int32_t *token_ids, int64_t num_tokens, const pa_block_hash_t *root,
                                   int32_t algo, pa_block_hash_t *out_hashes, int64_t *num_blocks)
{
    if (num_tokens < 0 || !num_blocks || (num_tokens > 0 && !token_ids))
        return PA_ERR_INVALID_ARG;
    if (algo != PA_HASH_FNV1A64 && algo != PA_HASH_SHA256)
        return PA_ERR_INVALID_ARG;
    const int64_t nb = num_tokens / kBlockTokens; // full blocks only
    *num_blocks = nb;
    if (nb == 0)
        return PA_OK;
    if (!out_hashes)
        return PA_ERR_INVALID_ARG;
    uint8_t parent[kDigest] = {};
    if (root)
        std::memcpy(parent, root->bytes, kDigest);
    for (int64_t b = 0; b < nb; ++b) {
        block_digest(parent, token_ids + b * kBlockTokens, algo, out_hashes[b].bytes);
        std::memcpy(parent, out_hashes[b].bytes, kDigest);
    }
    return PA_OK;
}

pa_prefix_cache_t *pa_prefix_cache_create(void) { return new (std::nothrow) pa_prefix_cache(); }

void pa_prefix_cache_destroy(pa_prefix_cache_t *cache) { delete cache; }

pa_status_t pa_prefix_cache_insert(pa_prefix_cache_t *cache, const pa_block_hash_t *hashes, const int32_t *block_ids,
                                   int32_t n)
{
    if (!cache || n < 0 || (n > 0 && (!hashes || !block_ids)))
        return PA_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i)
        if (block_ids[i] < 0)
            return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(cache->mu);
    for (int32_t i = 0; i < n; ++i) {
        std::string key(reinterpret_cast<const char *>(hashes[i].bytes), kDigest);
        if (cache->by_hash.count(key) || cache->by_block.count(block_ids[i]))
            continue; // first mapping wins; a block holds one hash until it is removed
        cache->by_hash.emplace(key, block_ids[i]);
        cache->by_block.emplace(block_ids[i], std::move(key));
    }
    return PA_OK;
}

pa_status_t pa_prefix_cache_remove_block(pa_prefix_cache_t *cache, int32_t block_id)
{
    if (!cache)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(cache->mu);
    auto it = cache->by_block.find(block_id);
    if (it != cache->by_block.end()) {
        cache->by_hash.erase(it->second);
        cache->by_block.erase(it);
    }
    return PA_OK;
}

int32_t pa_prefix_cache_longest_hit(pa_prefix_cache_t *cache, const pa_block_hash_t *hashes, int32_t n,
                                    int32_t *out_block_ids)
{
    if (!cache || n < 0 || (n > 0 && (!hashes || !out_block_ids)))
        return -1;
    std::lock_guard<std::mutex> g(cache->mu);
    int32_t hit = 0;
    for (; hit < n; ++hit) {
        auto it = cache->by_hash.find(std::string(reinterpret_cast<const char *>(hashes[hit].bytes), kDigest));
        if (it == cache->by_hash.end())
            break;
        out_block_ids[hit] = it->second;
    }
    return hit;
}

int64_t pa_prefix_cache_size(pa_prefix_cache_t *cache)
{
    if (!cache)
        return -1;
    std::lock_guard<std::mutex> g(cache->mu);
    return (int64_t)cache->by_hash.size();
}

} // extern "C"
