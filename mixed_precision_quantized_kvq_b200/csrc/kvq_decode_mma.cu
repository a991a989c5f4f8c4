// Host side of the persistent register-fragment decode kernel
// (kvq_decode_mma.cuh): which layouts it takes and its workspace.
#include "kvq_decode_mma_launch.cuh"

namespace kvq {

namespace {

template <int KB, int VB>
int slots_nh(const Params& p, int batch) {
    return p.g <= 4 ? mma::ring_slots<KB, VB, 4>(batch, p.g) : mma::ring_slots<KB, VB, 8>(batch, p.g);
}
template <int KB>
int slots_vb(const Params& p, int batch) {
    switch (p.vb) {
        case 1: return slots_nh<KB, 1>(p, batch);
        case 2: return slots_nh<KB, 2>(p, batch);
        case 4: return slots_nh<KB, 4>(p, batch);
        case 8: return slots_nh<KB, 8>(p, batch);
        default: return 0;
    }
}
int ring_slots_for(const Params& p, int batch) {
    switch (p.kb) {
        case 1: return slots_vb<1>(p, batch);
        case 2: return slots_vb<2>(p, batch);
        case 4: return slots_vb<4>(p, batch);
        case 8: return slots_vb<8>(p, batch);
        default: return 0;
    }
}

}  // namespace

bool mma_supported(const Params& p, int batch) {
    return p.d == mma::D && p.kg == 32 && p.vg == 128 && p.g >= 1 && p.g <= kMaxGqa && batch >= 1 &&
           batch <= mma::kMaxBatch && ring_slots_for(p, batch) > 0;
}

size_t mma_workspace_layout(const Params& p, int batch, int ctas, size_t* off_tickets) {
    const int nh = p.g <= 4 ? 4 : 8;
    const size_t part = (size_t(ctas) * 2 * nh * mma::PST * sizeof(float) + 255) & ~size_t(255);
    if (off_tickets) *off_tickets = part;
    return part + ((size_t(batch) * p.hkv * sizeof(uint32_t) + 255) & ~size_t(255));
}

}  // namespace kvq
