// Host-side planning of the expert-parallel exchange (no device code, no CUDA calls).
//
//  * exchange_schedule: a transmission order for one exchange with traffic matrix D in which no
//    two senders feed the same receiver at once, and whose length is the lower bound of
//    "MoE Inference Communication", §Aurora 定理 4.2: max over ranks of the tokens a rank sends
//    or receives over links. The pages' own procedure (Aurora, Algorithm 1: bottleneck rank
//    first, the others by volume, no receiver shared) only states the rule and the bound; here
//    the bound is reached by construction: D is embedded in a 2W x 2W matrix whose every row and
//    column sums to the bound, and that matrix is peeled into weighted permutations (Birkhoff's
//    decomposition; each permutation the one whose smallest entry is largest, found by
//    bisection over the values and augmenting paths, Kuhn's method). Each permutation
//    restricted to the real block is one phase.
//
//  * place_experts: which E/P experts of every layer each of P GPUs holds, so that few token
//    hops between consecutive layers cross GPUs ("MoE Inference Communication", §ExFlow
//    形式化：整数线性规划建模: the objective, the equal-share and one-GPU-per-expert
//    constraints). The pages solve it as an ILP; here it is solved by block coordinate descent:
//    the placement of one layer, given both neighbours, is a transportation problem (experts to
//    GPUs, E/P each) solved exactly by successive shortest paths, so every accepted move lowers
//    the cost; sweeps run forward and backward over the layers from several starts (one of
//    them groups the first layer's experts by the similarity of their affinity rows), and
//    each start's result is perturbed and descended again a few times (iterated local search).
//
//  * place_experts_staged: the staged form of the same page — experts on nodes first, then, node
//    by node, on that node's GPUs.
#pragma once

#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <vector>

namespace moe_plan {

// ------------------------------------------------------------------ exchange schedule

// Perfect matching on the entries >= thr (thr >= 1) of an n x n matrix (Kuhn's augmenting
// paths).
struct SupportMatching {
    int n;
    const std::vector<int64_t> &m;
    std::vector<int> row_to, col_to, seen;
    int stamp = 0;
    int64_t thr = 1;

    SupportMatching(int n_, const std::vector<int64_t> &m_)
        : n(n_), m(m_), row_to(n_, -1), col_to(n_, -1), seen(n_, -1) {}

    bool augment_from(int r)
    {
        for (int c = 0; c < n; ++c) {
            if (m[(size_t)r * n + c] < thr || seen[c] == stamp)
                continue;
            seen[c] = stamp;
            if (col_to[c] < 0 || augment_from(col_to[c])) {
                row_to[r] = c;
                col_to[c] = r;
                return true;
            }
        }
        return false;
    }

    bool match_row(int r)
    {
        ++stamp;
        return augment_from(r);
    }

    // A perfect matching from scratch on the entries >= t; false if there is none.
    bool match_all(int64_t t)
    {
        thr = t;
        std::fill(row_to.begin(), row_to.end(), -1);
        std::fill(col_to.begin(), col_to.end(), -1);
        for (int r = 0; r < n; ++r)
            if (!match_row(r))
                return false;
        return true;
    }
};

// Off-diagonal line sums of D and their maximum (the bound, in tokens).
inline int64_t exchange_bound(int W, const int64_t *D, std::vector<int64_t> *row,
                              std::vector<int64_t> *col)
{
    row->assign(W, 0);
    col->assign(W, 0);
    for (int i = 0; i < W; ++i)
        for (int j = 0; j < W; ++j)
            if (i != j) {
                (*row)[i] += D[i * W + j];
                (*col)[j] += D[i * W + j];
            }
    int64_t b = 0;
    for (int i = 0; i < W; ++i)
        b = std::max(b, std::max((*row)[i], (*col)[i]));
    return b;
}

// Returns false when the phases do not fit in max_phases (cannot happen for
// max_phases >= 2*W*W) or when no perfect matching exists (cannot happen for D >= 0).
// Each phase is the perfect matching of the remaining matrix whose smallest piece is largest
// (a bottleneck matching, found by bisection over the entries' values): few, long phases, as
// an executor pays one synchronisation per phase (a uniform 8-rank matrix: 32 phases where
// keeping one matching and repairing it as entries run out takes 95; 64 ranks: 218 against
// 7066). Every step still zeroes at least one entry, so there are at most 2*W*W of them.
inline bool exchange_schedule(int W, const int64_t *D, int max_phases, int32_t *phase_dst,
                              int64_t *phase_len, int *n_phases, int64_t *makespan)
{
    std::vector<int64_t> row, col;
    const int64_t bound = exchange_bound(W, D, &row, &col);
    *n_phases = 0;
    *makespan = 0;
    if (bound == 0)
        return true;
    // [ D_off            diag(bound - row) ]   every row and column of this 2W x 2W
    // [ diag(bound - col)     D_off^T       ]   matrix sums to `bound`.
    const int n = 2 * W;
    std::vector<int64_t> m((size_t)n * n, 0);
    for (int i = 0; i < W; ++i) {
        for (int j = 0; j < W; ++j)
            if (i != j) {
                m[(size_t)i * n + j] = D[i * W + j];
                m[(size_t)(W + j) * n + (W + i)] = D[i * W + j];
            }
        m[(size_t)i * n + (W + i)] = bound - row[i];
        m[(size_t)(W + i) * n + i] = bound - col[i];
    }
    SupportMatching pm(n, m);
    std::vector<int> best;
    std::vector<int64_t> vals;
    int64_t left = bound;
    while (left > 0) {
        vals.clear();
        for (int64_t v : m)
            if (v > 0)
                vals.push_back(v);
        std::sort(vals.begin(), vals.end());
        vals.erase(std::unique(vals.begin(), vals.end()), vals.end());
        int lo = 0, hi = (int)vals.size() - 1;
        best.clear();
        while (lo <= hi) {
            const int mid = (lo + hi) / 2;
            if (pm.match_all(vals[mid])) {
                best = pm.row_to;
                lo = mid + 1;
            } else {
                hi = mid - 1;
            }
        }
        if (best.empty())
            return false;
        int64_t step = left;
        for (int r = 0; r < n; ++r)
            step = std::min(step, m[(size_t)r * n + best[r]]);
        // The phase: sender i -> receiver best[i] when that entry lies in the real block.
        bool same = *n_phases > 0;
        for (int i = 0; i < W && same; ++i) {
            const int dst = best[i] < W ? best[i] : -1;
            same = phase_dst[(size_t)(*n_phases - 1) * W + i] == dst;
        }
        if (same) {
            phase_len[*n_phases - 1] += step;
        } else {
            if (*n_phases >= max_phases)
                return false;
            for (int i = 0; i < W; ++i)
                phase_dst[(size_t)*n_phases * W + i] = best[i] < W ? best[i] : -1;
            phase_len[*n_phases] = step;
            ++*n_phases;
        }
        for (int r = 0; r < n; ++r)
            m[(size_t)r * n + best[r]] -= step;
        left -= step;
        *makespan += step;
    }
    return true;
}

// ------------------------------------------------------------------ expert placement

// Experts to P GPUs, E / P each, maximising the summed score[e][q] (E x P, row-major): a
// transportation problem, solved exactly by successive shortest paths over the GPUs with
// potentials (the Hungarian method with capacitated columns). Experts enter one at a time; a
// Dijkstra over GPUs, reduced costs cost - u[e] - v[q] >= 0 (cost = -score), finds the cheapest
// way to seat the newcomer, possibly moving seated experts to other GPUs along the path; the
// potentials then keep every seated pair at reduced cost 0. O(E^2 P) in all, against O(E^3)
// for the square assignment with E/P copies of each GPU.
inline void balanced_assignment(int E, int P, const std::vector<int64_t> &score,
                                std::vector<int> *bin_of)
{
    const int share = E / P;
    std::vector<int64_t> u(E, 0), v(P, 0), dist(P);
    std::vector<int> prev_row(P), prev_bin(P), count(P, 0);
    std::vector<char> done(P);
    std::vector<std::vector<int>> members(P);
    bin_of->assign(E, -1);
    auto rc = [&](int e, int q) { return -score[(size_t)e * P + q] - u[e] - v[q]; };
    for (int s = 0; s < E; ++s) {
        for (int q = 0; q < P; ++q) {
            dist[q] = rc(s, q);
            prev_row[q] = s;
            prev_bin[q] = -1;
            done[q] = 0;
        }
        int t = -1;
        for (;;) {
            int q = -1;
            for (int k = 0; k < P; ++k)
                if (!done[k] && (q < 0 || dist[k] < dist[q]))
                    q = k;
            done[q] = 1;
            if (count[q] < share) {
                t = q;
                break;
            }
            for (int r : members[q])
                for (int k = 0; k < P; ++k) {
                    if (done[k])
                        continue;
                    const int64_t nd = dist[q] + rc(r, k);
                    if (nd < dist[k]) {
                        dist[k] = nd;
                        prev_row[k] = r;
                        prev_bin[k] = q;
                    }
                }
        }
        const int64_t delta = dist[t];
        for (int q = 0; q < P; ++q)
            if (done[q]) {
                v[q] -= delta - dist[q];
                for (int r : members[q])
                    u[r] += delta - dist[q];
            }
        u[s] += delta;
        // seat along the path: the row that reached t moves into t, and so on back to s
        for (int q = t;;) {
            const int r = prev_row[q];
            const int from = prev_bin[q];
            if (from >= 0) {
                auto &m = members[from];
                m.erase(std::find(m.begin(), m.end(), r));
                --count[from];
            }
            members[q].push_back(r);
            ++count[q];
            (*bin_of)[r] = q;
            if (r == s)
                break;
            q = from;
        }
    }
}

struct Placement {
    int L, E, P;
    const int64_t *counts;  // [L-1][E][E]

    int64_t cnt(int j, int i, int p) const { return counts[((size_t)j * E + i) * E + p]; }

    // Hops between consecutive layers whose experts sit on different GPUs.
    int64_t cost(const std::vector<int32_t> &g) const
    {
        int64_t c = 0;
        for (int j = 0; j + 1 < L; ++j)
            for (int i = 0; i < E; ++i)
                for (int p = 0; p < E; ++p)
                    if (g[(size_t)j * E + i] != g[(size_t)(j + 1) * E + p])
                        c += cnt(j, i, p);
        return c;
    }

    // Re-places layer l given its neighbours (only the previous layer when !right, and then
    // the result is taken even when it is not better); returns true if it changed the layer.
    bool improve_layer(int l, std::vector<int32_t> *g, bool right = true) const
    {
        std::vector<int64_t> score((size_t)E * P, 0);
        if (l > 0)
            for (int i = 0; i < E; ++i) {
                const int q = (*g)[(size_t)(l - 1) * E + i];
                for (int e = 0; e < E; ++e)
                    score[(size_t)e * P + q] += cnt(l - 1, i, e);
            }
        if (right && l + 1 < L)
            for (int e = 0; e < E; ++e)
                for (int p = 0; p < E; ++p)
                    score[(size_t)e * P + (*g)[(size_t)(l + 1) * E + p]] += cnt(l, e, p);
        int64_t current = 0;
        for (int e = 0; e < E; ++e)
            current += score[(size_t)e * P + (*g)[(size_t)l * E + e]];
        std::vector<int> bin;
        balanced_assignment(E, P, score, &bin);
        int64_t best = 0;
        for (int e = 0; e < E; ++e)
            best += score[(size_t)e * P + bin[e]];
        if (right && best <= current)
            return false;
        bool changed = false;
        for (int e = 0; e < E; ++e) {
            changed |= (*g)[(size_t)l * E + e] != bin[e];
            (*g)[(size_t)l * E + e] = bin[e];
        }
        return changed;
    }
};

// splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators", 2014).
inline uint64_t splitmix64(uint64_t *state)
{
    uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Layer 0's experts in P groups of E/P whose hops go to similar experts of layer 1 (cosine
// similarity of their rows of the affinity counts): P seeds taken farthest-first, then every
// other expert, most decided first, joins the group with room whose members it resembles
// most on average. Experts that feed the same experts next belong on the same GPU, and no
// single-layer move of the local search can gather them once they are spread.
inline void similarity_groups(int E, int P, const int64_t *c0, int32_t *group)
{
    const int share = E / P;
    std::vector<double> norm(E, 0.0), sim((size_t)E * E, 0.0);
    for (int i = 0; i < E; ++i) {
        double q = 0.0;
        for (int p = 0; p < E; ++p)
            q += (double)c0[(size_t)i * E + p] * (double)c0[(size_t)i * E + p];
        norm[i] = q > 0.0 ? std::sqrt(q) : 1.0;
    }
    for (int i = 0; i < E; ++i)
        for (int k = i; k < E; ++k) {
            double dot = 0.0;
            for (int p = 0; p < E; ++p)
                dot += (double)c0[(size_t)i * E + p] * (double)c0[(size_t)k * E + p];
            sim[(size_t)i * E + k] = sim[(size_t)k * E + i] = dot / (norm[i] * norm[k]);
        }
    std::vector<int> size(P, 0);
    std::vector<double> gsum((size_t)E * P, 0.0);  // expert x group: summed similarity
    for (int e = 0; e < E; ++e)
        group[e] = -1;
    auto join = [&](int e, int q) {
        group[e] = q;
        ++size[q];
        for (int k = 0; k < E; ++k)
            gsum[(size_t)k * P + q] += sim[(size_t)k * E + e];
    };
    // seeds: the expert with the most hops, then each time the one least like any seed
    int first = 0;
    for (int e = 1; e < E; ++e)
        if (norm[e] > norm[first])
            first = e;
    join(first, 0);
    for (int q = 1; q < P; ++q) {
        int pick = -1;
        double best = 0.0;
        for (int e = 0; e < E; ++e) {
            if (group[e] >= 0)
                continue;
            double closest = -1.0;
            for (int r = 0; r < q; ++r)
                closest = std::max(closest, gsum[(size_t)e * P + r]);
            if (pick < 0 || closest < best) {
                pick = e;
                best = closest;
            }
        }
        join(pick, q);
    }
    for (int left = E - P; left > 0; --left) {
        int pe = -1, pq = -1;
        double pv = 0.0;
        for (int e = 0; e < E; ++e) {
            if (group[e] >= 0)
                continue;
            for (int q = 0; q < P; ++q) {
                if (size[q] >= share)
                    continue;
                const double v = gsum[(size_t)e * P + q] / size[q];
                if (pe < 0 || v > pv) {
                    pe = e;
                    pq = q;
                    pv = v;
                }
            }
        }
        join(pe, pq);
    }
}

// Start 0: every layer contiguous (expert e on GPU e / (E/P)), so the result is never worse
// than that placement. Start 1: layer 0 contiguous. Start 2: layer 0 grouped by
// similarity_groups (set by the caller). Start s >= 3, with k = s - 1: layer 0 a shuffle of the
// contiguous assignment (Fisher-Yates driven by splitmix64 seeded with k); for odd k every
// other layer is shuffled the same way. Returns true when the later layers are still to be
// built from layer 0 (each placed best given the one before it).
inline bool initial_placement(int L, int E, int P, int start, std::vector<int32_t> *g)
{
    const int share = E / P;
    g->assign((size_t)L * E, 0);
    const int k = start - 1;  // the shuffle's seed and kind for start >= 3
    uint64_t state = (uint64_t)k;
    for (int l = 0; l < L; ++l) {
        int32_t *row = g->data() + (size_t)l * E;
        for (int e = 0; e < E; ++e)
            row[e] = e / share;
        if (start >= 3 && (l == 0 || k % 2 == 1))
            for (int e = E - 1; e > 0; --e) {
                const int r = (int)(splitmix64(&state) % (uint64_t)(e + 1));
                std::swap(row[e], row[r]);
            }
    }
    return start == 1 || start == 2 || (start >= 3 && k % 2 == 0);
}

// Block coordinate descent: each layer re-placed best given its neighbours, forward then
// backward, until a sweep changes nothing (at most 64 sweeps).
inline void descend(const Placement &pl, std::vector<int32_t> *g)
{
    for (int sweep = 0; sweep < 64 && pl.L > 1; ++sweep) {
        bool moved = false;
        for (int l = 0; l < pl.L; ++l)
            moved |= pl.improve_layer(l, g);
        for (int l = pl.L - 2; l > 0; --l)
            moved |= pl.improve_layer(l, g);
        if (!moved)
            break;
    }
}

inline void place_experts(int L, int E, int P, const int64_t *counts, int starts,
                          int32_t *gpu_of, int64_t *cost_out, int64_t *contiguous_out)
{
    const Placement pl{L, E, P, counts};
    std::vector<int32_t> best, g, h;
    int64_t best_cost = INT64_MAX;
    for (int s = 0; s < starts; ++s) {
        const bool build = initial_placement(L, E, P, s, &g);
        if (s == 0 && contiguous_out)
            *contiguous_out = pl.cost(g);
        if (s == 2 && L > 1 && P > 1)
            similarity_groups(E, P, counts, g.data());
        if (build)
            for (int l = 1; l < L; ++l)
                pl.improve_layer(l, &g, false);
        descend(pl, &g);
        int64_t c = pl.cost(g);
        // Kicks: swap the GPUs of two random pairs of experts in one layer, descend again,
        // keep the result if it is cheaper.
        uint64_t state = 0x5eedull + (uint64_t)s;
        for (int kick = 0; kick < 4 * L && L > 1 && P > 1; ++kick) {
            h = g;
            const int l = (int)(splitmix64(&state) % (uint64_t)L);
            for (int t = 0; t < 2; ++t) {
                const int a = (int)(splitmix64(&state) % (uint64_t)E);
                const int b = (int)(splitmix64(&state) % (uint64_t)E);
                std::swap(h[(size_t)l * E + a], h[(size_t)l * E + b]);
            }
            descend(pl, &h);
            const int64_t ch = pl.cost(h);
            if (ch < c) {
                c = ch;
                g.swap(h);
            }
        }
        if (c < best_cost) {
            best_cost = c;
            best = g;
        }
    }
    std::copy(best.begin(), best.end(), gpu_of);
    if (cost_out)
        *cost_out = best_cost;
}

// Hops between consecutive layers whose experts' groups differ, a group being g / per
// (per = 1: GPUs; per = GPUs per node: nodes).
inline int64_t crossing_hops(int L, int E, const int64_t *counts, const int32_t *g, int per)
{
    int64_t c = 0;
    for (int j = 0; j + 1 < L; ++j)
        for (int i = 0; i < E; ++i)
            for (int p = 0; p < E; ++p)
                if (g[(size_t)j * E + i] / per != g[(size_t)(j + 1) * E + p] / per)
                    c += counts[((size_t)j * E + i) * E + p];
    return c;
}

// Two stages, as ExFlow's staged expert affinity: first the experts of every layer are placed
// on nodes (E / nodes each), minimising the hops that cross nodes; then, node by node, that
// node's experts are placed on its GPUs, minimising the hops inside the node that cross GPUs
// (the affinity counts restricted to the node's experts of consecutive layers).
inline void place_experts_staged(int L, int E, int nodes, int gpn, const int64_t *counts,
                                 int starts, int32_t *gpu_of)
{
    std::vector<int32_t> node_of((size_t)L * E);
    place_experts(L, E, nodes, counts, starts, node_of.data(), nullptr, nullptr);
    const int Ep = E / nodes;
    std::vector<int32_t> members((size_t)L * Ep), local((size_t)L * Ep);
    std::vector<int64_t> sub((size_t)(L > 1 ? L - 1 : 0) * Ep * Ep);
    for (int n = 0; n < nodes; ++n) {
        for (int l = 0; l < L; ++l) {
            int k = 0;
            for (int e = 0; e < E; ++e)
                if (node_of[(size_t)l * E + e] == n)
                    members[(size_t)l * Ep + k++] = e;
        }
        for (int j = 0; j + 1 < L; ++j)
            for (int a = 0; a < Ep; ++a)
                for (int b = 0; b < Ep; ++b)
                    sub[((size_t)j * Ep + a) * Ep + b] =
                        counts[((size_t)j * E + members[(size_t)j * Ep + a]) * E +
                               members[(size_t)(j + 1) * Ep + b]];
        place_experts(L, Ep, gpn, sub.data(), starts, local.data(), nullptr, nullptr);
        for (int l = 0; l < L; ++l)
            for (int a = 0; a < Ep; ++a)
                gpu_of[(size_t)l * E + members[(size_t)l * Ep + a]] =
                    n * gpn + local[(size_t)l * Ep + a];
    }
}

}  // namespace moe_plan
