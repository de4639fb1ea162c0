// Prefix code of the codebook indices (host side): TurboQuant review (Jump2Paper),
// limitations paragraph (an optimal prefix code on the b = 4 indices averages about 3.8
// bits). The code is Huffman's code of the one-coordinate index law under Lemma 1, fixed per
// (d, b): merges take the two least probable nodes, ties to the lower node id (leaves
// 0..L-1, merged nodes L, L+1, ... in creation order); codewords are canonical (symbols in
// (length, symbol) order get consecutive integers).
#include <algorithm>
#include <cmath>
#include <queue>
#include <vector>

#include "internal.h"

namespace tq {

void index_law(int d, int L, const double* t, double* p);

int build_prefix_code(const tq_state* st, EntropyTable* tab) {
    const int L = 1 << st->b_mse;
    if (st->b_mse < 1) return TQ_EINVAL;
    std::vector<double> p(L);
    index_law(st->p.d, L, st->bounds.data(), p.data());
    // Huffman's merges
    using Node = std::pair<double, int>;   // (probability, id): smallest first
    std::priority_queue<Node, std::vector<Node>, std::greater<Node>> heap;
    for (int i = 0; i < L; ++i) heap.push({p[i], i});
    std::vector<int> parent(2 * L, -1);
    int next = L;
    while (heap.size() > 1) {
        Node a = heap.top();
        heap.pop();
        Node b = heap.top();
        heap.pop();
        parent[a.second] = parent[b.second] = next;
        heap.push({a.first + b.first, next});
        ++next;
    }
    const int root = heap.top().second;
    double mean = 0.0;
    int maxlen = 0;
    for (int i = 0; i < L; ++i) {
        int depth = 0;
        for (int n = i; n != root; n = parent[n]) ++depth;
        if (L == 1) depth = 1;
        tab->len[i] = depth;
        maxlen = std::max(maxlen, depth);
        mean += p[i] * depth;
    }
    if (maxlen > kMaxCodeLen) return TQ_EUNSUPPORTED;
    // canonical codewords in (length, symbol) order
    std::vector<int> order(L);
    for (int i = 0; i < L; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return tab->len[a] < tab->len[b]; });
    uint32_t code = 0;
    int prev = tab->len[order[0]];
    for (int l = 0; l <= kMaxCodeLen + 1; ++l) {
        tab->count[l] = 0;
        tab->first[l] = 0;
        tab->start[l] = 0;
    }
    for (int k = 0; k < L; ++k) {
        const int i = order[k];
        if (k > 0) code = (code + 1) << (tab->len[i] - prev);
        prev = tab->len[i];
        tab->word[i] = code;
        // the codeword bit-reversed: its first bit lands at the lowest stream position
        uint32_t r = 0;
        for (int j = 0; j < tab->len[i]; ++j) r |= ((code >> j) & 1u) << (tab->len[i] - 1 - j);
        tab->rword[i] = r;
        tab->sym[k] = i;
        if (tab->count[tab->len[i]]++ == 0) {
            tab->first[tab->len[i]] = code;
            tab->start[tab->len[i]] = k;
        }
    }
    tab->L = L;
    tab->maxlen = maxlen;
    tab->mean_bits = mean;
    return TQ_OK;
}

}  // namespace tq
