// Host block manager: FIFO free list, per-sequence block tables, slot mapping,
// reference counts and copy-on-write.
//
// Follows "LLM 推理引擎内部原理" §2.3 (Block 分配器): the free pool is a FIFO of
// block ids; a new request takes ceil(n / block_size) blocks; appending a token
// writes into the last block while it has room, else takes one block from the
// front of the free list; freed blocks go to the back. "vLLM PagedAttention 深度
// 解析" §4.1 adds sharing: forked samples point at the same physical blocks with
// a reference count, and the first write into a shared block copies it for the
// writer (old count - 1, new count 1); §4.2: a block returns to the pool when its
// count reaches 0.
//
// Swapping ("为什么PagedAttention能让大模型推理吞吐量提升数倍", section on
// scheduling and preemption; "vLLM PagedAttention 深度解析" §5.2): a second pool
// of host (CPU) blocks with its own free list and counts. swap_out moves a set of
// sequences' blocks to host blocks (each distinct block once, counts moved per
// reference, device blocks freed at 0) and yields the (device, host) block map
// for the copy; swap_in is the mirror image. All or nothing: a move that does
// not fit in the destination pool changes nothing.
//
// Each free list is a ring buffer of capacity num_blocks (each id is either in
// the ring or referenced, never both), so every call is O(1) per block.
#include <cstdint>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pkv.h"

namespace {

struct Seq {
    std::vector<int32_t> table;
    int64_t len = 0;
    bool swapped = false;           // table holds host block ids
};

struct Pool {
    std::vector<int32_t> ring;      // free list, FIFO
    size_t head = 0, count = 0;
    std::vector<int32_t> ref;

    bool init(int n, const int32_t* order) {
        ring.resize(n);
        ref.assign(n, 0);
        if (order) {
            std::vector<char> seen(n, 0);
            for (int i = 0; i < n; ++i) {
                const int32_t b = order[i];
                if (b < 0 || b >= n || seen[b]) return false;
                seen[b] = 1;
                ring[i] = b;
            }
        } else {
            for (int i = 0; i < n; ++i) ring[i] = i;
        }
        head = 0;
        count = n;
        return true;
    }
    int size() const { return (int)ref.size(); }
    bool take(int32_t* b) {
        if (count == 0) return false;
        *b = ring[head];
        head = (head + 1) % ring.size();
        --count;
        ref[*b] = 1;
        return true;
    }
    void give_back(int32_t b) {
        ring[(head + count) % ring.size()] = b;
        ++count;
    }
    void release(int32_t b) {
        if (--ref[b] == 0) give_back(b);
    }
};

}  // namespace

struct pkv_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    Pool dev, host;
    std::unordered_map<int64_t, Seq> seqs;

    bool take(int32_t* b) { return dev.take(b); }
    void release(int32_t b) { dev.release(b); }
    size_t free_count() const { return dev.count; }
    int64_t slot(const Seq& s, int64_t pos) const {
        return (int64_t)s.table[pos / block_size] * block_size + pos % block_size;
    }
    // A resident sequence, or nullptr (unknown or swapped out).
    Seq* resident(int64_t id) {
        auto it = seqs.find(id);
        return (it == seqs.end() || it->second.swapped) ? nullptr : &it->second;
    }

    // Moves the listed sequences' blocks from pool `from` to pool `to`.
    pkv_status move(const int64_t* ids, int n, bool out, int64_t* src_out, int64_t* dst_out, int capacity,
                    int* num_pairs) {
        Pool& from = out ? dev : host;
        Pool& to = out ? host : dev;
        std::unordered_map<int32_t, int32_t> fresh;       // source block -> destination block
        std::unordered_map<int64_t, char> listed;
        for (int i = 0; i < n; ++i) {
            auto it = seqs.find(ids[i]);
            if (it == seqs.end() || it->second.swapped != !out || listed.count(ids[i]))
                return PKV_ERR_INVALID_ARG;
            listed[ids[i]] = 1;
            for (int32_t b : it->second.table) fresh.emplace(b, -1);
        }
        if (fresh.size() > (size_t)capacity) return PKV_ERR_INVALID_ARG;
        if (fresh.size() > to.count) return PKV_ERR_OUT_OF_BLOCKS;
        int np = 0;
        for (int i = 0; i < n; ++i) {
            Seq& s = seqs[ids[i]];
            for (int32_t& b : s.table) {
                int32_t& d = fresh[b];
                if (d < 0) {                                  // first sight: one copy
                    to.take(&d);
                    to.ref[d] = 0;
                    src_out[np] = b;
                    dst_out[np] = d;
                    ++np;
                }
                to.ref[d] += 1;
                from.release(b);
                b = d;
            }
            s.swapped = out;
        }
        *num_pairs = np;
        return PKV_OK;
    }
};

extern "C" {

pkv_status pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                         pkv_block_manager** out) {
    if (!out || num_blocks <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
    *out = nullptr;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
    if (!bm) return PKV_ERR_INVALID_ARG;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    if (!bm->dev.init(num_blocks, free_order)) { delete bm; return PKV_ERR_INVALID_ARG; }
    *out = bm;
    return PKV_OK;
}

pkv_status pkv_bm_set_host_pool(pkv_block_manager* bm, int num_host_blocks, const int32_t* free_order) {
    if (!bm || num_host_blocks < 0 || bm->host.size() > 0) return PKV_ERR_INVALID_ARG;
    if (num_host_blocks == 0) return PKV_OK;
    Pool p;
    if (!p.init(num_host_blocks, free_order)) return PKV_ERR_INVALID_ARG;
    bm->host = std::move(p);
    return PKV_OK;
}

pkv_status pkv_bm_swap_out(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* dev_blocks_out,
                           int64_t* host_blocks_out, int capacity, int* num_pairs_out) {
    if (num_pairs_out) *num_pairs_out = 0;
    if (!bm || n < 0 || capacity < 0 || !num_pairs_out ||
        (n > 0 && (!seq_ids || (capacity > 0 && (!dev_blocks_out || !host_blocks_out)))))
        return PKV_ERR_INVALID_ARG;
    return bm->move(seq_ids, n, true, dev_blocks_out, host_blocks_out, capacity, num_pairs_out);
}

pkv_status pkv_bm_swap_in(pkv_block_manager* bm, const int64_t* seq_ids, int n, int64_t* host_blocks_out,
                          int64_t* dev_blocks_out, int capacity, int* num_pairs_out) {
    if (num_pairs_out) *num_pairs_out = 0;
    if (!bm || n < 0 || capacity < 0 || !num_pairs_out ||
        (n > 0 && (!seq_ids || (capacity > 0 && (!dev_blocks_out || !host_blocks_out)))))
        return PKV_ERR_INVALID_ARG;
    return bm->move(seq_ids, n, false, host_blocks_out, dev_blocks_out, capacity, num_pairs_out);
}

int pkv_bm_num_free_host(const pkv_block_manager* bm) { return bm ? (int)bm->host.count : -1; }

int pkv_bm_host_ref_count(const pkv_block_manager* bm, int block) {
    if (!bm || block < 0 || block >= bm->host.size()) return -1;
    return bm->host.ref[block];
}

int pkv_bm_is_swapped(const pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (it->second.swapped ? 1 : 0);
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, int num_tokens, int64_t* slots_out) {
    if (!bm || num_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (bm->seqs.count(seq_id)) return PKV_ERR_INVALID_ARG;
    const int64_t nblk = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
    if ((size_t)nblk > bm->free_count()) return PKV_ERR_OUT_OF_BLOCKS;
    Seq s;
    s.table.resize(nblk);
    for (int64_t i = 0; i < nblk; ++i) bm->take(&s.table[i]);
    s.len = num_tokens;
    if (slots_out)
        for (int64_t p = 0; p < num_tokens; ++p) slots_out[p] = bm->slot(s, p);
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int64_t* slot_mapping_out, int64_t* copy_src_out,
                               int64_t* copy_dst_out, int* num_copies_out, int* num_done_out) {
    if (num_done_out) *num_done_out = 0;
    if (num_copies_out) *num_copies_out = 0;
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !slot_mapping_out || !copy_src_out ||
                                   !copy_dst_out || !num_copies_out)))
        return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!bm->resident(seq_ids[i])) return PKV_ERR_INVALID_ARG;
    int ncopy = 0;
    for (int i = 0; i < n; ++i) {
        Seq& s = bm->seqs[seq_ids[i]];
        const int64_t len = s.len;
        if (len % bm->block_size != 0) {
            int32_t last = s.table.back();
            if (bm->dev.ref[last] > 1) {         // shared partially filled block: copy-on-write
                int32_t fresh;
                if (!bm->take(&fresh)) { *num_copies_out = ncopy; return PKV_ERR_OUT_OF_BLOCKS; }
                bm->dev.ref[last] -= 1;
                s.table.back() = fresh;
                copy_src_out[ncopy] = last;
                copy_dst_out[ncopy] = fresh;
                ++ncopy;
            }
        } else {
            int32_t fresh;
            if (!bm->take(&fresh)) { *num_copies_out = ncopy; return PKV_ERR_OUT_OF_BLOCKS; }
            s.table.push_back(fresh);
        }
        slot_mapping_out[i] = bm->slot(s, len);
        s.len = len + 1;
        if (num_done_out) *num_done_out = i + 1;
    }
    *num_copies_out = ncopy;
    return PKV_OK;
}

pkv_status pkv_bm_make_writable(pkv_block_manager* bm, int64_t seq_id, int logical_block,
                                int64_t* src, int64_t* dst) {
    if (!bm || !src || !dst) return PKV_ERR_INVALID_ARG;
    *src = *dst = -1;
    Seq* sp = bm->resident(seq_id);
    if (!sp) return PKV_ERR_INVALID_ARG;
    Seq& s = *sp;
    if (logical_block < 0 || (size_t)logical_block >= s.table.size()) return PKV_ERR_INVALID_ARG;
    int32_t old = s.table[logical_block];
    if (bm->dev.ref[old] <= 1) return PKV_OK;
    int32_t fresh;
    if (!bm->take(&fresh)) return PKV_ERR_OUT_OF_BLOCKS;
    bm->dev.ref[old] -= 1;
    s.table[logical_block] = fresh;
    *src = old;
    *dst = fresh;
    return PKV_OK;
}

pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    Seq* p = bm->resident(parent);
    if (!p || bm->seqs.count(child)) return PKV_ERR_INVALID_ARG;
    Seq c = *p;
    for (int32_t b : c.table) bm->dev.ref[b] += 1;
    bm->seqs.emplace(child, std::move(c));
    return PKV_OK;
}

pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PKV_ERR_INVALID_ARG;
    Pool& pool = it->second.swapped ? bm->host : bm->dev;
    for (int32_t b : it->second.table) pool.release(b);
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int max_blocks, int32_t* tables_out, int32_t* context_lens_out) {
    if (!bm || n < 0 || max_blocks <= 0 || (n > 0 && (!seq_ids || !tables_out)))
        return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end() || it->second.swapped) return PKV_ERR_INVALID_ARG;
        const Seq& s = it->second;
        if (s.table.size() > (size_t)max_blocks || s.len > INT32_MAX) return PKV_ERR_INVALID_ARG;
        int32_t* row = tables_out + (size_t)i * max_blocks;
        std::memcpy(row, s.table.data(), s.table.size() * sizeof(int32_t));
        std::memset(row + s.table.size(), 0, (max_blocks - s.table.size()) * sizeof(int32_t));
        if (context_lens_out) context_lens_out[i] = (int32_t)s.len;
    }
    return PKV_OK;
}

int pkv_bm_block_size(const pkv_block_manager* bm) { return bm ? bm->block_size : -1; }

int pkv_bm_num_free(const pkv_block_manager* bm) { return bm ? (int)bm->dev.count : -1; }

int pkv_bm_ref_count(const pkv_block_manager* bm, int block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->dev.ref[block];
}

int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (int)it->second.len;
}

}  // extern "C"
