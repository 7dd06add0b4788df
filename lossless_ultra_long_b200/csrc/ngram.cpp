// ngram.cpp -- the n-gram reuse table of include/ts_verify.h (host code).
//
// TokenSwift reuses phrases that recur in the generated text as draft
// candidates and refreshes their frequencies after every verification
// ("TokenSwift - A framework for accelerating the generation of ultra-long
// text", aiboss88.com, "Parallel generation of multiple tokens and token
// reuse"; "TokenSwift ... 从小时到分钟", cloud.tencent.com, the
// parallel-verification step of the method figure).  The table lives in one
// caller-owned buffer:
//
//   Header | Slot[capacity] | Key[capacity] (first token) | Key[capacity] ((n-1)-prefix)
//
// A Slot holds one n-gram and its count (count 0 = empty); slots are found
// by open addressing with linear probing on a hash of the n tokens.  Two
// indices chain the slots: by first token (whole-phrase continuations of a
// token) and by the first n-1 tokens (next-token counts after a prefix).  A
// Key holds the head of one chain (-1 = empty entry; the key's tokens are
// read from its head slot) and that chain's best kTop slots in retrieval
// order.  Counts only grow, one at a time, so a best list stays exact when
// each counted slot is moved up in it (or enters it past its last entry);
// a retrieval of up to kTop n-grams on an indexed prefix reads the list and
// never walks the chain.  Nothing is ever removed.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "ts_verify.h"

namespace {

constexpr uint32_t kMagic = 0x4e475432u;   // "NGT2"
constexpr int kMaxN = 8;
constexpr int kMaxK = 4096;
constexpr int kTop = 16;                              // best n-grams kept per key
constexpr int64_t kMaxCapacity = int64_t(1) << 31;    // slot indices fit int32

struct Header {
    uint32_t magic;
    int32_t n;
    int64_t capacity;
    int64_t used;    // distinct n-grams held
    int64_t keys;    // distinct first tokens held
    int64_t total;   // n-grams counted, with multiplicity
    int64_t reserved[3];
};
static_assert(sizeof(Header) == 64, "header is 64 bytes");

struct Slot {
    int32_t tok[kMaxN];
    int64_t count;
    int64_t next[2];   // next slot in the chain of index 0 / 1, -1 at the end
};
static_assert(sizeof(Slot) == 56, "slot is 56 bytes");

struct Key {
    int64_t head;        // -1: empty entry
    int32_t n_top;       // entries of top[] in use
    int32_t pad;
    int32_t top[kTop];   // best slots of the chain, retrieval order
};
static_assert(sizeof(Key) == 80, "key is 80 bytes");

bool capacity_ok(int64_t c) { return c >= 2 && c <= kMaxCapacity && (c & (c - 1)) == 0; }

size_t table_bytes(int n, int64_t capacity)
{
    if (n < 2 || n > kMaxN || !capacity_ok(capacity))
        return 0;
    return sizeof(Header) + (size_t)capacity * (sizeof(Slot) + 2 * sizeof(Key));
}

// At least one slot stays empty, so every probe sequence ends.
int64_t fill_limit(int64_t capacity) { return capacity - std::max<int64_t>(1, capacity / 8); }

// FNV-1a (64-bit) over the little-endian bytes of the tokens, folded so the
// high half reaches the low bits that index the table.
uint64_t hash_tokens(const int32_t *t, int n)
{
    uint64_t h = 14695981039346656037ull;
    for (int i = 0; i < n; ++i) {
        const uint32_t v = (uint32_t)t[i];
        for (int b = 0; b < 4; ++b) {
            h ^= (v >> (8 * b)) & 0xffu;
            h *= 1099511628211ull;
        }
    }
    return h ^ (h >> 32);
}

struct View {
    Header *hdr;
    Slot *slots;
    Key *keys[2];   // index 0: first token; index 1: first n-1 tokens
    int n;
    int64_t mask;
    int plen(int idx) const { return idx == 0 ? 1 : n - 1; }
};

// The table in `p` if it is formatted and fits in `bytes`.
bool view_of(const void *p, size_t bytes, View &v)
{
    if (!p || (reinterpret_cast<uintptr_t>(p) & 7) != 0 || bytes < sizeof(Header))
        return false;
    Header *h = static_cast<Header *>(const_cast<void *>(p));
    if (h->magic != kMagic || table_bytes(h->n, h->capacity) == 0 ||
        bytes < table_bytes(h->n, h->capacity))
        return false;
    v.hdr = h;
    v.slots = reinterpret_cast<Slot *>(h + 1);
    v.keys[0] = reinterpret_cast<Key *>(v.slots + h->capacity);
    v.keys[1] = v.keys[0] + h->capacity;
    v.n = h->n;
    v.mask = h->capacity - 1;
    return true;
}

// Slot holding gram, or the empty slot where it would go.
int64_t find_slot(const View &v, const int32_t *gram)
{
    int64_t i = (int64_t)(hash_tokens(gram, v.n) & (uint64_t)v.mask);
    for (;;) {
        const Slot &s = v.slots[i];
        if (s.count == 0 || memcmp(s.tok, gram, sizeof(int32_t) * v.n) == 0)
            return i;
        i = (i + 1) & v.mask;   // the fill limit keeps an empty slot on every probe path
    }
}

// Key of index `idx` for the prefix (its first plen tokens), or the empty
// entry where it would go.  Keys never outnumber slots.
int64_t find_key(const View &v, int idx, const int32_t *prefix)
{
    const int p = v.plen(idx);
    const Key *keys = v.keys[idx];
    int64_t i = (int64_t)(hash_tokens(prefix, p) & (uint64_t)v.mask);
    for (;;) {
        const Key &k = keys[i];
        if (k.head < 0 || memcmp(v.slots[k.head].tok, prefix, sizeof(int32_t) * p) == 0)
            return i;
        i = (i + 1) & v.mask;
    }
}

// lexicographic order of two token runs of length n
bool tokens_less(const int32_t *a, const int32_t *b, int n)
{
    for (int i = 0; i < n; ++i)
        if (a[i] != b[i])
            return a[i] < b[i];
    return false;
}

// Retrieval order of two slots that share a prefix: count descending, then
// the tokens after the first in ascending order (for a shared prefix of any
// length that is the order of the continuations).
bool ranks_before(const View &v, int64_t a, int64_t b)
{
    const Slot &x = v.slots[a], &y = v.slots[b];
    if (x.count != y.count)
        return x.count > y.count;
    return tokens_less(x.tok + 1, y.tok + 1, v.n - 1);
}

// slot s of key k's chain was just counted: keep k's best list exact
void refresh_top(const View &v, Key &k, int32_t s)
{
    int pos = -1;
    for (int i = 0; i < k.n_top; ++i)
        if (k.top[i] == s) {
            pos = i;
            break;
        }
    if (pos < 0) {
        if (k.n_top < kTop)
            pos = k.n_top++;
        else if (ranks_before(v, s, k.top[kTop - 1]))
            pos = kTop - 1;
        else
            return;
        k.top[pos] = s;
    }
    for (; pos > 0 && ranks_before(v, k.top[pos], k.top[pos - 1]); --pos) {
        const int32_t t = k.top[pos];
        k.top[pos] = k.top[pos - 1];
        k.top[pos - 1] = t;
    }
}

}  // namespace

extern "C" {

size_t ts_ngram_table_bytes(int n, int64_t capacity) { return table_bytes(n, capacity); }

int ts_ngram_init(void *table, size_t bytes, int n, int64_t capacity)
{
    const size_t need = table_bytes(n, capacity);
    if (!table || need == 0 || bytes < need || (reinterpret_cast<uintptr_t>(table) & 7) != 0)
        return TS_ERR_INVALID_ARG;
    Header *h = static_cast<Header *>(table);
    memset(h, 0, sizeof(Header));
    Slot *slots = reinterpret_cast<Slot *>(h + 1);
    Key *keys = reinterpret_cast<Key *>(slots + capacity);
    memset(slots, 0, sizeof(Slot) * (size_t)capacity);
    memset(keys, 0, 2 * sizeof(Key) * (size_t)capacity);
    for (int64_t i = 0; i < 2 * capacity; ++i)
        keys[i].head = -1;
    h->n = n;
    h->capacity = capacity;
    h->magic = kMagic;
    return TS_OK;
}

int ts_ngram_update(void *table, size_t bytes, const int32_t *text, int64_t text_len,
                    int64_t n_new)
{
    View v;
    if (!view_of(table, bytes, v) || text_len < 0 || n_new < 0 || n_new > text_len ||
        (text_len > 0 && !text))
        return TS_ERR_INVALID_ARG;
    const int n = v.n;
    // n-grams ending at positions [e0, text_len)
    const int64_t e0 = std::max<int64_t>(n - 1, text_len - n_new);
    if (e0 >= text_len)
        return TS_OK;
    for (int64_t p = e0 - (n - 1); p < text_len; ++p)
        if (text[p] < 0)
            return TS_ERR_INVALID_ARG;

    // distinct n-grams not yet in the table: all or nothing
    std::vector<int64_t> fresh;   // start positions
    try {
        for (int64_t e = e0; e < text_len; ++e) {
            const int32_t *g = text + e - (n - 1);
            if (v.slots[find_slot(v, g)].count == 0)
                fresh.push_back(e - (n - 1));
        }
        std::sort(fresh.begin(), fresh.end(), [&](int64_t a, int64_t b) {
            return tokens_less(text + a, text + b, n);
        });
    } catch (const std::bad_alloc &) {
        return TS_ERR_WORKSPACE;
    }
    int64_t distinct = 0;
    for (size_t i = 0; i < fresh.size(); ++i)
        if (i == 0 || memcmp(text + fresh[i - 1], text + fresh[i], sizeof(int32_t) * n) != 0)
            ++distinct;
    if (v.hdr->used + distinct > fill_limit(v.hdr->capacity))
        return TS_ERR_WORKSPACE;

    for (int64_t e = e0; e < text_len; ++e) {
        const int32_t *g = text + e - (n - 1);
        const int64_t si = find_slot(v, g);
        Slot &s = v.slots[si];
        Key *k[2] = {&v.keys[0][find_key(v, 0, g)], &v.keys[1][find_key(v, 1, g)]};
        if (s.count == 0) {
            // the tokens first: an empty key found above is compared
            // against its head slot's tokens from now on
            memset(s.tok, 0, sizeof(s.tok));
            memcpy(s.tok, g, sizeof(int32_t) * n);
            for (int idx = 0; idx < 2; ++idx) {
                if (k[idx]->head < 0) {
                    k[idx]->n_top = 0;
                    if (idx == 0)
                        ++v.hdr->keys;
                }
                s.next[idx] = k[idx]->head;
                k[idx]->head = si;
            }
            ++v.hdr->used;
        }
        ++s.count;
        ++v.hdr->total;
        refresh_top(v, *k[0], (int32_t)si);
        refresh_top(v, *k[1], (int32_t)si);
    }
    return TS_OK;
}

int ts_ngram_topk_prefix(const void *table, size_t bytes, const int32_t *prefix, int p, int k,
                         int32_t *cont_out, int64_t *count_out, int *n_found)
{
    View v;
    if (!view_of(table, bytes, v) || !prefix || p < 1 || p > v.n - 1 || k < 1 || k > kMaxK ||
        !cont_out || !count_out || !n_found)
        return TS_ERR_INVALID_ARG;
    const int m = v.n - p;   // continuation tokens per row
    for (int i = 0; i < k; ++i) {
        count_out[i] = 0;
        for (int j = 0; j < m; ++j)
            cont_out[(size_t)i * m + j] = -1;
    }
    *n_found = 0;
    for (int i = 0; i < p; ++i)
        if (prefix[i] < 0)
            return TS_OK;   // no such n-gram can be held
    // an indexed prefix length walks (or reads the best list of) its own
    // chain; any other walks the first-token chain and filters
    const int idx = p == 1 ? 0 : (p == v.n - 1 ? 1 : 0);
    const bool filter = p != v.plen(idx);
    const Key &key = v.keys[idx][find_key(v, idx, prefix)];
    if (key.head < 0)
        return TS_OK;
    auto emit = [&](const int64_t *slots, int found) {
        for (int i = 0; i < found; ++i) {
            const Slot &s = v.slots[slots[i]];
            count_out[i] = s.count;
            memcpy(cont_out + (size_t)i * m, s.tok + p, sizeof(int32_t) * m);
        }
        *n_found = found;
    };
    // the best list holds the whole chain while it is not full, and the
    // chain's best kTop once it is
    if (!filter && (k <= key.n_top || key.n_top < kTop)) {
        int64_t top[kTop];
        const int found = k < key.n_top ? k : key.n_top;
        for (int i = 0; i < found; ++i)
            top[i] = key.top[i];
        emit(top, found);
        return TS_OK;
    }
    // walk the chain, keeping the best k sorted in the same order
    int found = 0;
    std::vector<int64_t> best;
    try {
        best.reserve((size_t)k);
    } catch (const std::bad_alloc &) {
        return TS_ERR_WORKSPACE;
    }
    for (int64_t s = key.head; s >= 0; s = v.slots[s].next[idx]) {
        if (filter && memcmp(v.slots[s].tok, prefix, sizeof(int32_t) * p) != 0)
            continue;
        if (found == k && !ranks_before(v, s, best[k - 1]))
            continue;
        if (found < k) {
            best.push_back(s);
            ++found;
        } else {
            best[k - 1] = s;
        }
        for (int i = found - 1; i > 0 && ranks_before(v, best[i], best[i - 1]); --i)
            std::swap(best[i], best[i - 1]);
    }
    emit(best.data(), found);
    return TS_OK;
}

int ts_ngram_topk(const void *table, size_t bytes, int32_t first, int k, int32_t *cont_out,
                  int64_t *count_out, int *n_found)
{
    return ts_ngram_topk_prefix(table, bytes, &first, 1, k, cont_out, count_out, n_found);
}

int ts_ngram_count(const void *table, size_t bytes, const int32_t *gram, int64_t *count)
{
    View v;
    if (!view_of(table, bytes, v) || !gram || !count)
        return TS_ERR_INVALID_ARG;
    *count = v.slots[find_slot(v, gram)].count;
    return TS_OK;
}

int ts_ngram_size(const void *table, size_t bytes, int64_t *distinct, int64_t *total)
{
    View v;
    if (!view_of(table, bytes, v) || !distinct || !total)
        return TS_ERR_INVALID_ARG;
    *distinct = v.hdr->used;
    *total = v.hdr->total;
    return TS_OK;
}

}  // extern "C"
