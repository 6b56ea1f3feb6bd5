// slot_cache.cpp -- host-side slot allocator and radix-tree prefix cache for
// GDN state slots (contract: gdn_slot_cache.h).
//
// This is the logical cache layer of the pages' hybrid prefix cache (24-ai.news
// TokenSpeed article, "Hybrid prefix caching for GDN/Mamba": a C++ logical cache,
// radix-tree matching with state-slot extensions, copy-on-write reuse; zubnet.ai
// LightSeek TokenSpeed article, second paragraph: checkpoints reused without
// mutation, speculative decoding through current_input_indices).  It decides slot
// numbers only; the device sees them as gdn_decode_step / gdn_commit index tables.

#include "gdn_slot_cache.h"

#include <cstdint>
#include <memory>
#include <new>
#include <set>
#include <unordered_map>
#include <utility>
#include <vector>

namespace {

struct Node {
    std::vector<int32_t> label;  // tokens on the edge from the parent
    Node* parent = nullptr;
    std::unordered_map<int32_t, std::unique_ptr<Node>> children;  // keyed by the child's first label token
    int64_t depth = 0;     // tokens from the root to the end of this node
    int32_t slot = -1;     // checkpoint: slot holding the state after this node's prefix
    uint64_t last_use = 0;
};

struct Request {
    bool open = false;
    int32_t slot = -1;             // slot holding the current state
    int32_t plan_T = 0;            // 0: no pending plan
    std::vector<int32_t> planned;  // destination slots of the pending plan (T entries)
};

}  // namespace

struct gdn_slot_cache {
    int32_t num_slots = 0;
    std::vector<int32_t> ref;       // holders per slot: requests + checkpoints
    std::vector<int32_t> tree_ref;  // the checkpoints among them
    std::vector<int32_t> free_list;
    Node root;
    uint64_t tick = 0;
    std::set<std::pair<uint64_t, Node*>> lru;  // checkpoint nodes by last use
    int32_t checkpoints = 0;
    std::vector<Request> reqs;
    std::vector<int32_t> free_reqs;
    int32_t open_requests = 0;

    // Tear the tree down iteratively: a chain of checkpoints one token apart
    // could otherwise recurse as deep as the longest cached context.
    ~gdn_slot_cache() {
        std::vector<std::unique_ptr<Node>> stack;
        for (auto& kv : root.children) stack.push_back(std::move(kv.second));
        root.children.clear();
        while (!stack.empty()) {
            std::unique_ptr<Node> n = std::move(stack.back());
            stack.pop_back();
            for (auto& kv : n->children) stack.push_back(std::move(kv.second));
            n->children.clear();
        }
    }

    bool valid_slot(int32_t s) const { return s >= 0 && s < num_slots; }
    bool valid_req(int32_t r) const { return r >= 0 && r < (int32_t)reqs.size() && reqs[r].open; }

    void retain(int32_t s) { ++ref[s]; }
    void release(int32_t s) {
        if (--ref[s] == 0) free_list.push_back(s);
    }

    void touch(Node* n) {
        lru.erase({n->last_use, n});
        n->last_use = ++tick;
        lru.insert({n->last_use, n});
    }

    // Drops empty leaves upward from n (never the root).
    void prune(Node* n) {
        while (n != &root && n->slot < 0 && n->children.empty()) {
            Node* p = n->parent;
            p->children.erase(n->label[0]);  // destroys n
            n = p;
        }
    }

    // Evicts the least recently used checkpoint whose slot no request holds.
    // (Several checkpoints may name one slot; the slot is freed with the last.)
    bool evict_one() {
        for (auto it = lru.begin(); it != lru.end(); ++it) {
            Node* n = it->second;
            if (ref[n->slot] != tree_ref[n->slot]) continue;  // a request still reads it
            lru.erase(it);
            const int32_t s = n->slot;
            n->slot = -1;
            --checkpoints;
            --tree_ref[s];
            release(s);
            prune(n);
            return true;
        }
        return false;
    }

    // Slots that evictions could free: each distinct checkpoint slot that no
    // request holds (all of its holders are checkpoints).
    int64_t evictable_slots() const {
        std::set<int32_t> slots;
        for (const auto& e : lru) {
            const int32_t s = e.second->slot;
            if (ref[(size_t)s] == tree_ref[(size_t)s]) slots.insert(s);
        }
        return (int64_t)slots.size();
    }

    // A free slot with reference count 1, evicting if needed; -1 if none.  One eviction
    // frees nothing when another checkpoint names the same slot, so evict until a slot is
    // free.  Every evictable checkpoint's slot is held by checkpoints only, so the loop
    // ends with a free slot whenever evictable_slots() > 0, and evicts nothing otherwise.
    int32_t alloc() {
        while (free_list.empty())
            if (!evict_one()) return -1;
        const int32_t s = free_list.back();
        free_list.pop_back();
        ref[s] = 1;
        return s;
    }

    // Deepest checkpoint whose whole prefix lies inside tokens[0..n).
    Node* match(const int32_t* tokens, int64_t n) {
        Node* cur = &root;
        Node* best = nullptr;
        int64_t i = 0;
        while (i < n) {
            auto it = cur->children.find(tokens[i]);
            if (it == cur->children.end()) break;
            Node* ch = it->second.get();
            size_t m = 0;
            while (m < ch->label.size() && i + (int64_t)m < n && ch->label[m] == tokens[i + m]) ++m;
            if (m < ch->label.size()) break;  // the context ends inside this edge, or diverges in it
            cur = ch;
            i += (int64_t)m;
            if (cur->slot >= 0) best = cur;
        }
        return best;
    }

    // The node for exactly tokens[0..n), created (splitting an edge if needed).
    Node* insert_path(const int32_t* tokens, int64_t n) {
        Node* cur = &root;
        int64_t i = 0;
        while (i < n) {
            auto it = cur->children.find(tokens[i]);
            if (it == cur->children.end()) {
                auto leaf = std::make_unique<Node>();
                leaf->label.assign(tokens + i, tokens + n);
                leaf->parent = cur;
                leaf->depth = n;
                Node* p = leaf.get();
                cur->children.emplace(tokens[i], std::move(leaf));
                return p;
            }
            Node* ch = it->second.get();
            size_t m = 0;
            while (m < ch->label.size() && i + (int64_t)m < n && ch->label[m] == tokens[i + m]) ++m;
            if (m == ch->label.size()) {
                cur = ch;
                i += (int64_t)m;
                continue;
            }
            // Split ch's edge after m tokens: cur -> mid -> ch.
            auto mid = std::make_unique<Node>();
            mid->label.assign(ch->label.begin(), ch->label.begin() + (std::ptrdiff_t)m);
            mid->parent = cur;
            mid->depth = cur->depth + (int64_t)m;
            std::unique_ptr<Node> held = std::move(it->second);
            held->label.erase(held->label.begin(), held->label.begin() + (std::ptrdiff_t)m);
            held->parent = mid.get();
            const int32_t key = held->label[0];
            mid->children.emplace(key, std::move(held));
            Node* midp = mid.get();
            it->second = std::move(mid);
            cur = midp;
            i += (int64_t)m;
        }
        return cur;
    }
};

extern "C" {

gdn_status gdn_slot_cache_create(int32_t num_slots, gdn_slot_cache** cache) {
    try {
        if (cache == nullptr || num_slots < 1) return GDN_ERR_INVALID_ARG;
        std::unique_ptr<gdn_slot_cache> c(new gdn_slot_cache());
        c->num_slots = num_slots;
        c->ref.assign((size_t)num_slots, 0);
        c->tree_ref.assign((size_t)num_slots, 0);
        c->free_list.reserve((size_t)num_slots);
        for (int32_t s = num_slots - 1; s >= 0; --s) c->free_list.push_back(s);  // slot 0 handed out first
        *cache = c.release();
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

void gdn_slot_cache_destroy(gdn_slot_cache* cache) { delete cache; }

gdn_status gdn_slot_cache_open(gdn_slot_cache* c, const int32_t* tokens, int64_t n, int32_t* req, int32_t* slot,
                               int64_t* matched_len, int32_t* needs_init) {
    try {
        if (c == nullptr || n < 0 || (n > 0 && tokens == nullptr) || req == nullptr || slot == nullptr ||
            matched_len == nullptr || needs_init == nullptr)
            return GDN_ERR_INVALID_ARG;
        Node* hit = c->match(tokens, n);
        int32_t s;
        if (hit != nullptr) {
            s = hit->slot;
            c->retain(s);
            c->touch(hit);
            *matched_len = hit->depth;
            *needs_init = 0;
        } else {
            s = c->alloc();
            if (s < 0) return GDN_ERR_CAPACITY;
            *matched_len = 0;
            *needs_init = 1;
        }
        int32_t id;
        if (!c->free_reqs.empty()) {
            id = c->free_reqs.back();
            c->free_reqs.pop_back();
        } else {
            id = (int32_t)c->reqs.size();
            c->reqs.emplace_back();
        }
        Request& r = c->reqs[(size_t)id];
        r.open = true;
        r.slot = s;
        r.plan_T = 0;
        r.planned.clear();
        ++c->open_requests;
        *req = id;
        *slot = s;
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_plan(gdn_slot_cache* c, const int32_t* reqs, int32_t B, int32_t T, int32_t* src_idx,
                               int32_t* dst_idx) {
    try {
        if (c == nullptr || B < 0 || T < 1 || (B > 0 && (reqs == nullptr || src_idx == nullptr || dst_idx == nullptr)))
            return GDN_ERR_INVALID_ARG;
        std::set<int32_t> seen;
        for (int32_t b = 0; b < B; ++b) {
            if (!c->valid_req(reqs[b]) || c->reqs[(size_t)reqs[b]].plan_T != 0 || !seen.insert(reqs[b]).second)
                return GDN_ERR_INVALID_ARG;
        }
        // Count the fresh slots first: the plan fails before it takes a slot or
        // evicts a checkpoint, so a failing call changes nothing.  Taking slots
        // never changes which requests own theirs, nor which checkpoints are
        // evictable (the planned requests hold their own slots), so the count is exact.
        int64_t fresh = 0;
        for (int32_t b = 0; b < B; ++b) {
            const Request& r = c->reqs[(size_t)reqs[b]];
            fresh += (T == 1 && c->ref[(size_t)r.slot] == 1) ? 0 : T;
        }
        if (fresh > (int64_t)c->free_list.size() &&
            fresh > (int64_t)c->free_list.size() + c->evictable_slots())
            return GDN_ERR_CAPACITY;
        std::vector<int32_t> taken;  // fresh slots of this plan, returned if it fails
        for (int32_t b = 0; b < B; ++b) {
            Request& r = c->reqs[(size_t)reqs[b]];
            src_idx[b] = r.slot;
            for (int32_t t = 0; t < T; ++t) {
                int32_t d;
                if (T == 1 && c->ref[(size_t)r.slot] == 1) {
                    d = r.slot;  // owned: update in place
                } else {
                    d = c->alloc();  // shared (copy-on-write fork) or a draft slot
                    if (d < 0) {
                        for (int32_t s : taken) c->release(s);
                        for (int32_t bb = 0; bb < b; ++bb) {
                            Request& rr = c->reqs[(size_t)reqs[bb]];
                            rr.plan_T = 0;
                            rr.planned.clear();
                        }
                        r.planned.clear();
                        return GDN_ERR_CAPACITY;
                    }
                    taken.push_back(d);
                }
                dst_idx[(size_t)b * T + t] = d;
                r.planned.push_back(d);
            }
            r.plan_T = T;
        }
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_commit(gdn_slot_cache* c, const int32_t* reqs, int32_t B, int32_t T,
                                 const int32_t* accept_len, int32_t* committed) {
    try {
        if (c == nullptr || B < 0 || T < 1 || (B > 0 && reqs == nullptr) || (T > 1 && B > 0 && accept_len == nullptr))
            return GDN_ERR_INVALID_ARG;
        std::set<int32_t> seen;
        for (int32_t b = 0; b < B; ++b) {
            if (!c->valid_req(reqs[b]) || c->reqs[(size_t)reqs[b]].plan_T != T || !seen.insert(reqs[b]).second)
                return GDN_ERR_INVALID_ARG;
            if (T > 1 && (accept_len[b] < 0 || accept_len[b] > T)) return GDN_ERR_INVALID_ARG;
        }
        for (int32_t b = 0; b < B; ++b) {
            Request& r = c->reqs[(size_t)reqs[b]];
            const int32_t a = T == 1 ? 1 : accept_len[b];
            if (a >= 1) {
                const int32_t keep = r.planned[(size_t)(a - 1)];
                if (keep != r.slot) c->release(r.slot);
                r.slot = keep;
            }
            for (int32_t t = 0; t < T; ++t) {
                const int32_t d = r.planned[(size_t)t];
                if (t != a - 1 && d != r.slot) c->release(d);  // rejected drafts
            }
            r.planned.clear();
            r.plan_T = 0;
            if (committed != nullptr) committed[b] = r.slot;
        }
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_checkpoint(gdn_slot_cache* c, int32_t req, const int32_t* tokens, int64_t n,
                                     int32_t* slot) {
    try {
        if (c == nullptr || !c->valid_req(req) || n < 1 || tokens == nullptr) return GDN_ERR_INVALID_ARG;
        Request& r = c->reqs[(size_t)req];
        if (r.plan_T != 0) return GDN_ERR_INVALID_ARG;  // the state is mid-step
        Node* node = c->insert_path(tokens, n);
        if (node->slot < 0) {
            node->slot = r.slot;
            c->retain(r.slot);
            ++c->tree_ref[(size_t)r.slot];
            ++c->checkpoints;
        }
        c->touch(node);
        if (slot != nullptr) *slot = node->slot;
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_close(gdn_slot_cache* c, int32_t req) {
    try {
        if (c == nullptr || !c->valid_req(req)) return GDN_ERR_INVALID_ARG;
        Request& r = c->reqs[(size_t)req];
        for (int32_t d : r.planned)
            if (d != r.slot) c->release(d);
        c->release(r.slot);
        r = Request();
        c->free_reqs.push_back(req);
        --c->open_requests;
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_evict(gdn_slot_cache* c, int32_t want_free, int32_t* evicted) {
    try {
        if (c == nullptr || want_free < 0) return GDN_ERR_INVALID_ARG;
        int32_t n = 0;
        while ((int32_t)c->free_list.size() < want_free && c->evict_one()) ++n;
        if (evicted != nullptr) *evicted = n;
        return GDN_OK;
    } catch (...) {  // no C++ exception crosses the C ABI
        return GDN_ERR_CAPACITY;
    }
}

gdn_status gdn_slot_cache_stats(const gdn_slot_cache* c, int32_t* free_slots, int32_t* checkpoints,
                                int32_t* open_requests) {
    if (c == nullptr) return GDN_ERR_INVALID_ARG;
    if (free_slots != nullptr) *free_slots = (int32_t)c->free_list.size();
    if (checkpoints != nullptr) *checkpoints = c->checkpoints;
    if (open_requests != nullptr) *open_requests = c->open_requests;
    return GDN_OK;
}

int32_t gdn_slot_cache_refcount(const gdn_slot_cache* c, int32_t slot) {
    if (c == nullptr || !c->valid_slot(slot)) return -1;
    return c->ref[(size_t)slot];
}

}  // extern "C"
