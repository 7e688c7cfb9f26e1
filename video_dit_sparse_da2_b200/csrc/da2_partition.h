// da2_partition.h -- host region partition of a video frame (see the .cpp).
#pragma once
#include <vector>

namespace da2 {

struct FramePartition {
    int Rf = 0;               // regions (= 64-token blocks) per frame
    int bands = 0;            // band count of the chosen candidate
    std::vector<int> region;  // [Hv*Wv] region of each cell (row-major)
    std::vector<int> slot;    // [Hv*Wv] position of the cell inside its region
    std::vector<int> size;    // [Rf] valid cells per region
};

bool build_partition(int Hv, int Wv, int C, FramePartition* out);

}  // namespace da2
