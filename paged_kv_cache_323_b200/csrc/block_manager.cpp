// block_manager.cpp -- host-side block manager (include/pkv_block_manager.h):
// free lists of device and host blocks, per-sequence block tables, reference
// counts, forks, copy-on-write decisions, release on finish, swapping, and
// the counters.  Plain C++; every device copy it asks for is run by the
// caller through copy_blocks / swap_blocks.
#include <stdint.h>

#include <algorithm>
#include <new>
#include <vector>

#include "../../include/pkv_block_manager.h"

struct pkv_block_manager {
    struct Seq {
        std::vector<int32_t> blocks;       // device blocks, logical order
        std::vector<int32_t> host_blocks;  // host blocks while swapped out
        int64_t length = 0;
        int64_t arrival = 0;
        bool live = false;     // resident on the device
        bool swapped = false;  // blocks held in the host pool
    };

    int num_blocks = 0;
    int block_size = 0;
    int num_host_blocks = 0;
    std::vector<int32_t> free_dev;   // stack: back() is handed out next
    std::vector<int32_t> free_host;  // stack
    std::vector<int32_t> ref;        // refcount per device block
    std::vector<Seq> seqs;
    int64_t next_arrival = 0;
    int64_t preemptions = 0;
    int64_t cow_pairs = 0;

    bool valid_seq(int s) const { return s >= 0 && s < (int)seqs.size(); }

    int32_t take_dev() {
        const int32_t b = free_dev.back();
        free_dev.pop_back();
        ref[b] = 1;
        return b;
    }

    void release_dev(int32_t b) {
        if (--ref[b] == 0) free_dev.push_back(b);
    }

    int blocks_for(int64_t len) const { return (int)((len + block_size - 1) / block_size); }
};

namespace {

bool room(int64_t* pairs, int max_pairs, int need) { return need <= max_pairs && (need == 0 || pairs); }

}  // namespace

extern "C" {

pkv_block_manager* pkv_bm_create(int num_blocks, int block_size, int num_host_blocks,
                                 const int32_t* free_order) {
    if (num_blocks <= 0 || block_size <= 0 || num_host_blocks < 0) return nullptr;
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
    if (!bm) return nullptr;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->num_host_blocks = num_host_blocks;
    bm->ref.assign(num_blocks, 0);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return nullptr;  // not a permutation
            }
            seen[b] = 1;
        }
    }
    bm->free_dev.resize(num_blocks);
    for (int i = 0; i < num_blocks; ++i)  // the stack pops from the back: reverse the order
        bm->free_dev[num_blocks - 1 - i] = free_order ? free_order[i] : i;
    bm->free_host.resize(num_host_blocks);
    for (int i = 0; i < num_host_blocks; ++i) bm->free_host[num_host_blocks - 1 - i] = i;
    return bm;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

int pkv_bm_add_sequence(pkv_block_manager* bm) {
    if (!bm) return PKV_ERR_NULL;
    pkv_block_manager::Seq s;
    s.live = true;
    s.arrival = bm->next_arrival++;
    bm->seqs.push_back(s);
    return (int)bm->seqs.size() - 1;
}

int pkv_bm_fork(pkv_block_manager* bm, int parent) {
    if (!bm) return PKV_ERR_NULL;
    if (!bm->valid_seq(parent) || !bm->seqs[parent].live) return PKV_ERR_INVALID;
    pkv_block_manager::Seq child;
    child.blocks = bm->seqs[parent].blocks;
    child.length = bm->seqs[parent].length;
    child.live = true;
    child.arrival = bm->next_arrival++;
    for (int32_t b : child.blocks) ++bm->ref[b];
    bm->seqs.push_back(child);
    return (int)bm->seqs.size() - 1;
}

int pkv_bm_append(pkv_block_manager* bm, int seq, int n, int64_t* slots, int64_t* cow_pairs,
                  int max_pairs, int* n_pairs) {
    if (!bm || !n_pairs || (n > 0 && !slots)) return PKV_ERR_NULL;
    if (!bm->valid_seq(seq) || !bm->seqs[seq].live || n < 0) return PKV_ERR_INVALID;
    *n_pairs = 0;
    if (n == 0) return PKV_OK;
    pkv_block_manager::Seq& s = bm->seqs[seq];
    const int bs = bm->block_size;
    const int have = (int)s.blocks.size();
    const int need = bm->blocks_for(s.length + n);
    // copy-on-write: the first new token goes into a partly filled, shared last block
    const bool partial_last = s.length % bs != 0;
    const bool cow = partial_last && bm->ref[s.blocks.back()] > 1;
    const int fresh = (need - have) + (cow ? 1 : 0);
    if (fresh > (int)bm->free_dev.size()) return PKV_ERR_OUT_OF_BLOCKS;
    if (cow && !room(cow_pairs, max_pairs, 1)) return PKV_ERR_INVALID;
    if (cow) {
        const int32_t src = s.blocks.back();
        const int32_t dst = bm->take_dev();
        bm->release_dev(src);
        s.blocks.back() = dst;
        cow_pairs[0] = src;
        cow_pairs[1] = dst;
        *n_pairs = 1;
        ++bm->cow_pairs;
    }
    while ((int)s.blocks.size() < need) s.blocks.push_back(bm->take_dev());
    for (int i = 0; i < n; ++i) {
        const int64_t t = s.length + i;
        slots[i] = (int64_t)s.blocks[t / bs] * bs + t % bs;
    }
    s.length += n;
    return PKV_OK;
}

int pkv_bm_free(pkv_block_manager* bm, int seq) {
    if (!bm) return PKV_ERR_NULL;
    if (!bm->valid_seq(seq)) return PKV_ERR_INVALID;
    pkv_block_manager::Seq& s = bm->seqs[seq];
    if (!s.live && !s.swapped) return PKV_ERR_INVALID;
    for (int32_t b : s.blocks) bm->release_dev(b);
    for (int32_t h : s.host_blocks) bm->free_host.push_back(h);
    s.blocks.clear();
    s.host_blocks.clear();
    s.live = s.swapped = false;
    s.length = 0;
    return PKV_OK;
}

int pkv_bm_tables(const pkv_block_manager* bm, const int32_t* seqs, int n, int max_blocks,
                  int32_t* tables, int32_t* context_lens) {
    if (!bm || (n > 0 && (!seqs || !tables || !context_lens))) return PKV_ERR_NULL;
    if (n < 0 || max_blocks <= 0) return PKV_ERR_INVALID;
    for (int i = 0; i < n; ++i) {
        if (!bm->valid_seq(seqs[i]) || !bm->seqs[seqs[i]].live) return PKV_ERR_INVALID;
        if ((int)bm->seqs[seqs[i]].blocks.size() > max_blocks) return PKV_ERR_INVALID;
    }
    for (int i = 0; i < n; ++i) {
        const pkv_block_manager::Seq& s = bm->seqs[seqs[i]];
        int32_t* row = tables + (int64_t)i * max_blocks;
        std::fill(row, row + max_blocks, -1);
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        context_lens[i] = (int32_t)s.length;
    }
    return PKV_OK;
}

int pkv_bm_length(const pkv_block_manager* bm, int seq) {
    if (!bm) return PKV_ERR_NULL;
    if (!bm->valid_seq(seq) || (!bm->seqs[seq].live && !bm->seqs[seq].swapped)) return PKV_ERR_INVALID;
    return (int)bm->seqs[seq].length;
}

int pkv_bm_pick_victim(const pkv_block_manager* bm) {
    if (!bm) return PKV_ERR_NULL;
    int best = -1;
    for (int i = 0; i < (int)bm->seqs.size(); ++i)
        if (bm->seqs[i].live && (best < 0 || bm->seqs[i].arrival > bm->seqs[best].arrival)) best = i;
    return best;
}

int pkv_bm_swap_out(pkv_block_manager* bm, int seq, int64_t* pairs, int max_pairs, int* n_pairs) {
    if (!bm || !n_pairs) return PKV_ERR_NULL;
    if (!bm->valid_seq(seq) || !bm->seqs[seq].live) return PKV_ERR_INVALID;
    pkv_block_manager::Seq& s = bm->seqs[seq];
    const int nb = (int)s.blocks.size();
    if (nb > (int)bm->free_host.size()) return PKV_ERR_OUT_OF_BLOCKS;
    if (!room(pairs, max_pairs, nb)) return PKV_ERR_INVALID;
    s.host_blocks.clear();
    for (int j = 0; j < nb; ++j) {
        const int32_t h = bm->free_host.back();
        bm->free_host.pop_back();
        s.host_blocks.push_back(h);
        pairs[2 * j] = s.blocks[j];
        pairs[2 * j + 1] = h;
    }
    // the copies are enqueued before any later use of the released device
    // blocks, on the same stream, so the blocks can be handed out again now
    for (int32_t b : s.blocks) bm->release_dev(b);
    s.blocks.clear();
    s.live = false;
    s.swapped = true;
    *n_pairs = nb;
    ++bm->preemptions;
    return PKV_OK;
}

int pkv_bm_swap_in(pkv_block_manager* bm, int seq, int64_t* pairs, int max_pairs, int* n_pairs) {
    if (!bm || !n_pairs) return PKV_ERR_NULL;
    if (!bm->valid_seq(seq) || !bm->seqs[seq].swapped) return PKV_ERR_INVALID;
    pkv_block_manager::Seq& s = bm->seqs[seq];
    const int nb = (int)s.host_blocks.size();
    if (nb > (int)bm->free_dev.size()) return PKV_ERR_OUT_OF_BLOCKS;
    if (!room(pairs, max_pairs, nb)) return PKV_ERR_INVALID;
    s.blocks.clear();
    for (int j = 0; j < nb; ++j) {
        const int32_t d = bm->take_dev();
        s.blocks.push_back(d);
        pairs[2 * j] = s.host_blocks[j];
        pairs[2 * j + 1] = d;
    }
    for (int32_t h : s.host_blocks) bm->free_host.push_back(h);
    s.host_blocks.clear();
    s.swapped = false;
    s.live = true;
    *n_pairs = nb;
    return PKV_OK;
}

int pkv_bm_get_stats(const pkv_block_manager* bm, pkv_bm_stats* out) {
    if (!bm || !out) return PKV_ERR_NULL;
    pkv_bm_stats st = {};
    st.num_blocks = bm->num_blocks;
    st.free_blocks = (int64_t)bm->free_dev.size();
    st.host_free_blocks = (int64_t)bm->free_host.size();
    st.preemptions = bm->preemptions;
    st.copy_on_write = bm->cow_pairs;
    // per physical block: how many of its slots hold a token of some sequence
    std::vector<int32_t> filled(bm->num_blocks, 0);
    const int bs = bm->block_size;
    for (const pkv_block_manager::Seq& s : bm->seqs) {
        if (s.swapped) ++st.swapped_sequences;
        if (!s.live) continue;
        ++st.live_sequences;
        st.logical_allocated += (int64_t)s.blocks.size() * bs;
        st.logical_used += s.length;
        for (size_t j = 0; j < s.blocks.size(); ++j) {
            const int64_t here = std::min<int64_t>(bs, s.length - (int64_t)j * bs);
            filled[s.blocks[j]] = std::max<int32_t>(filled[s.blocks[j]], (int32_t)here);
        }
    }
    for (int b = 0; b < bm->num_blocks; ++b) {
        if (bm->ref[b] > 0) {
            ++st.used_blocks;
            st.used_slots += filled[b];
        }
    }
    st.allocated_slots = st.used_blocks * bs;
    *out = st;
    return PKV_OK;
}

}  // extern "C"
