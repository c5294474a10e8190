// The exhibit's allocation bench, on the host ("KV 缓存与分页注意力" §实验台):
// requests arrive one after another, write their prompt at once, then one
// token per round, and leave when done; those that do not fit wait.  The
// memory is either paged (blocks of block_size slots from the block manager)
// or reserved up front as one contiguous run per request: max_len slots (the
// exhibit's "max" setting, §先占好最长的位置), or the two other reservations
// the paper's Orca baselines use (§三种浪费): the next power of two of the
// final length, or exactly the final length.  Readouts: rounds to finish all,
// peak concurrency, how much of the held memory holds tokens, and the held
// slots split into reservation (written later) and internal fragmentation
// (never written); all taken each round after admission and writing, before
// the finished requests leave.
//
// Rules taken where the page is silent:
// * Round r: (1) admission, first come first served in arrival order, a
//   request that does not fit stops admission for the round; (2) every request
//   admitted in an earlier round writes one token; (3) finished requests leave.
// * "max": first-fit contiguous run of max_len slots.
// * Paged growth that finds no free block preempts the most recently admitted
//   running request (§放不下的时候: the latest to start gives up all of its
//   blocks); it returns to the head of the waiting queue and is later
//   recomputed: its prompt plus the tokens it had written become its new
//   prompt.  A request may preempt itself.
#include <algorithm>
#include <deque>
#include <vector>

#include "block_manager.h"
#include "pagedkv.h"

namespace {

struct Live {
    int id;
    int written;      // tokens stored
    int total;        // prompt + output
    int admitted;     // round of admission
    long long order;  // admission sequence number (latest = largest)
    int slot0;        // contiguous modes: first reserved slot
    int held;         // contiguous modes: slots reserved
};

int reservation(const pkv_sim_request& r, int mode, int max_len) {
    const int total = r.prompt + r.output;
    if (mode == PKV_SIM_MAX) return max_len;
    if (mode == PKV_SIM_ORACLE) return total;
    int p = 1;
    while (p < total) p *= 2;
    return p < max_len ? p : max_len;
}

}  // namespace

extern "C" pkv_status pkv_simulate(const pkv_sim_request* reqs, int n, int num_slots,
                                   int block_size, int max_len, int max_rounds,
                                   pkv_sim_result* out, int32_t* running_per_round) {
    if (!reqs || n < 0 || num_slots < 1 || block_size < PKV_SIM_ORACLE || max_len < 1 ||
        max_rounds < 1 || !out)
        return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const pkv_sim_request& r = reqs[i];
        if (r.arrival < 0 || r.prompt < 1 || r.output < 1 || r.prompt + r.output > max_len)
            return PKV_ERR_INVALID_ARG;
        if (i > 0 && r.arrival < reqs[i - 1].arrival) return PKV_ERR_INVALID_ARG;
    }
    if (block_size > 0 && num_slots % block_size) return PKV_ERR_INVALID_ARG;
    const bool paged = block_size > 0;
    pkv::BlockManager bm(paged ? num_slots / block_size : 1, paged ? block_size : 1);
    std::vector<char> slot_used(paged ? 0 : num_slots, 0);

    std::deque<std::pair<int, int>> waiting;   // (request, tokens already generated)
    int next_arrival = 0;
    std::vector<Live> running;
    long long admissions = 0;
    pkv_sim_result res{};
    std::vector<int> generated(n, 0);
    int finished = 0;
    double util_sum = 0.0;
    int util_rounds = 0;
    int round = 0;
    for (; round < max_rounds && finished < n; ++round) {
        while (next_arrival < n && reqs[next_arrival].arrival <= round)
            waiting.emplace_back(next_arrival++, 0);
        // (1) admission
        while (!waiting.empty()) {
            const int id = waiting.front().first;
            const int done = waiting.front().second;   // tokens generated before a preemption
            const int prompt = reqs[id].prompt + done;
            Live l{id, prompt, reqs[id].prompt + reqs[id].output, round, admissions, -1, 0};
            if (paged) {
                std::vector<int32_t> slots((size_t)prompt);
                if (bm.alloc(id, prompt, slots.data()) != PKV_OK) break;
            } else {
                const int want = reservation(reqs[id], block_size, max_len);
                int start = -1;
                for (int s = 0, run = 0; s < num_slots; ++s) {
                    run = slot_used[s] ? 0 : run + 1;
                    if (run == want) {
                        start = s - want + 1;
                        break;
                    }
                }
                if (start < 0) break;
                std::fill(slot_used.begin() + start, slot_used.begin() + start + want, 1);
                l.slot0 = start;
                l.held = want;
            }
            ++admissions;
            ++res.admitted;
            running.push_back(l);
            waiting.pop_front();
        }
        // (2) one token for every request admitted before this round
        for (size_t i = 0; i < running.size();) {
            if (running[i].admitted == round || running[i].written >= running[i].total) {
                ++i;
                continue;
            }
            const int cur = running[i].id;   // entries may move when a victim leaves
            if (paged) {
                int32_t slot, src, dst;
                bool self_preempted = false;
                while (bm.append(cur, &slot, &src, &dst) != PKV_OK) {
                    // preempt the latest admitted request
                    size_t victim = 0;
                    for (size_t j = 1; j < running.size(); ++j)
                        if (running[j].order > running[victim].order) victim = j;
                    const Live v = running[victim];
                    bm.release(v.id);
                    generated[v.id] = v.written - reqs[v.id].prompt;
                    waiting.emplace_front(v.id, generated[v.id]);
                    ++res.preemptions;
                    running.erase(running.begin() + victim);
                    if (v.id == cur) {
                        self_preempted = true;
                        break;
                    }
                    if (victim < i) --i;
                }
                if (self_preempted) continue;   // running[i] is now the next request
            }
            ++running[i].written;
            ++i;
        }
        // readouts of the round, while every request that wrote in it still
        // holds its memory
        long long stored = 0, reserved = 0;
        for (const Live& l : running) {
            const long long held =
                paged ? (long long)((l.written + block_size - 1) / block_size) * block_size : l.held;
            const long long will = std::min<long long>(held, l.total);
            stored += l.written;
            reserved += held;
            res.future_slot_rounds += will - l.written;
            res.internal_frag_slot_rounds += held - will;
        }
        res.peak_running = std::max(res.peak_running, (int32_t)running.size());
        res.stored_token_rounds += stored;
        res.reserved_slot_rounds += reserved;
        if (reserved > 0) {
            util_sum += (double)stored / (double)reserved;
            ++util_rounds;
        }
        if (running_per_round) running_per_round[round] = (int32_t)running.size();
        // (3) finished requests leave
        for (size_t i = 0; i < running.size();) {
            if (running[i].written >= running[i].total) {
                if (paged) {
                    bm.release(running[i].id);
                } else {
                    std::fill(slot_used.begin() + running[i].slot0,
                              slot_used.begin() + running[i].slot0 + running[i].held, 0);
                }
                ++finished;
                running.erase(running.begin() + i);
            } else {
                ++i;
            }
        }
    }
    if (finished < n) return PKV_ERR_INVALID_ARG;   // max_rounds too small
    res.rounds = round;
    res.mean_utilisation = util_rounds ? util_sum / util_rounds : 0.0;
    *out = res;
    return PKV_OK;
}
