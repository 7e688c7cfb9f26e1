// da2_partition.cpp -- host construction of the per-frame region partition
// ("DraftAttention2", Sec. 3.3 "Fused quantization and reordering"; App. C.2).
//
// The paper asks for a ragged 2-D partition of every frame into connected
// regions with balanced token counts bounded by the block capacity C, the
// minimum number of blocks R_f = ceil(Hv*Wv/C) (less than one block of
// padding per frame), and the smallest total perimeter among the candidate
// partitions.  App. C.2 is cut off on the page before it names the candidate
// family, so this file takes the following reading:
//   * region sizes: n/R_f rounded, the first (n mod R_f) regions one larger;
//   * candidates: for every band count nb = 1..Hv, rows split into nb bands of
//     balanced height (taller bands first), visited as a boustrophedon (even
//     bands left to right, odd bands right to left), each band column by
//     column with the vertical direction alternating per column; the visit
//     order is cut into consecutive chunks of the region sizes;
//   * keep candidates whose regions are all 4-connected (if none is, keep
//     all), pick the smallest total perimeter, ties to the smaller nb.
// A token's slot inside its block is its position in the visit order.
#include "da2_partition.h"

#include <algorithm>
#include <numeric>
#include <vector>

namespace da2 {

namespace {

struct UnionFind {
    std::vector<int> parent;
    explicit UnionFind(int n) : parent(n) { std::iota(parent.begin(), parent.end(), 0); }
    int find(int x) {
        while (parent[x] != x) x = parent[x] = parent[parent[x]];
        return x;
    }
    void join(int a, int b) { parent[find(a)] = find(b); }
};

// Visit order of the cells of an Hv x Wv frame for a given band count.
std::vector<int> band_visit(int Hv, int Wv, int nb) {
    std::vector<int> order;
    order.reserve((size_t)Hv * Wv);
    int y0 = 0;
    for (int band = 0; band < nb; ++band) {
        const int height = Hv / nb + (band < Hv % nb ? 1 : 0);
        for (int col = 0; col < Wv; ++col) {
            const int x = (band & 1) ? Wv - 1 - col : col;
            for (int r = 0; r < height; ++r) {
                const int y = (col & 1) ? y0 + height - 1 - r : y0 + r;
                order.push_back(y * Wv + x);
            }
        }
        y0 += height;
    }
    return order;
}

}  // namespace

bool build_partition(int Hv, int Wv, int C, FramePartition* out) {
    if (Hv <= 0 || Wv <= 0 || C <= 0) return false;
    const int n = Hv * Wv;
    const int Rf = (n + C - 1) / C;
    std::vector<int> size(Rf);
    for (int j = 0; j < Rf; ++j) size[j] = n / Rf + (j < n % Rf ? 1 : 0);

    auto label = [&](const std::vector<int>& order, std::vector<int>& region, std::vector<int>& slot) {
        region.assign(n, 0);
        slot.assign(n, 0);
        size_t pos = 0;
        for (int j = 0; j < Rf; ++j)
            for (int s = 0; s < size[j]; ++s, ++pos) {
                region[order[pos]] = j;
                slot[order[pos]] = s;
            }
    };

    int best_nb = -1;
    long best_perimeter = 0;
    bool best_connected = false;
    std::vector<int> region, slot;
    for (int nb = 1; nb <= Hv; ++nb) {
        label(band_visit(Hv, Wv, nb), region, slot);
        // Cut edges between different regions; connectivity by union-find.
        UnionFind uf(n);
        long cut = 0;
        for (int y = 0; y < Hv; ++y)
            for (int x = 0; x < Wv; ++x) {
                const int c = y * Wv + x;
                if (x + 1 < Wv) {
                    if (region[c + 1] == region[c]) uf.join(c, c + 1);
                    else ++cut;
                }
                if (y + 1 < Hv) {
                    if (region[c + Wv] == region[c]) uf.join(c, c + Wv);
                    else ++cut;
                }
            }
        std::vector<int> root_of_region(Rf, -1);
        bool connected = true;
        for (int c = 0; c < n && connected; ++c) {
            const int r = uf.find(c);
            int& seen = root_of_region[region[c]];
            if (seen < 0) seen = r;
            else if (seen != r) connected = false;
        }
        // Total perimeter: frame border plus both sides of every cut edge.
        const long perimeter = 2L * (Hv + Wv) + 2L * cut;
        const bool better = best_nb < 0 || (connected && !best_connected) ||
                            (connected == best_connected && perimeter < best_perimeter);
        if (better) {
            best_nb = nb;
            best_perimeter = perimeter;
            best_connected = connected;
        }
    }
    label(band_visit(Hv, Wv, best_nb), region, slot);
    out->Rf = Rf;
    out->bands = best_nb;
    out->region = region;
    out->slot = slot;
    out->size = size;
    return true;
}

}  // namespace da2
