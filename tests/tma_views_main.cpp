// Prints the TMA views that the expert-FFN kernels build over their weight tensors, for
// the sizes given on the command line (E I H), one line per view:
//   name rank elem_bytes dims[rank] strides[rank-1] box[rank]
// so that a host test can check footprints and row orders without a GPU.  Built with
// the host compiler against the library's own tmap.cuh (no driver call is made).
#include <cstdio>
#include <cstdlib>

#include "tmap.cuh"

using moe::tmap::View;

static void print(const char* name, bool ok, const View& v) {
    if (!ok) {
        std::printf("%s refused\n", name);
        return;
    }
    std::printf("%s %d %d", name, v.rank, v.elem_bytes);
    for (int d = 0; d < v.rank; ++d) std::printf(" %llu", static_cast<unsigned long long>(v.dims[d]));
    for (int d = 0; d + 1 < v.rank; ++d)
        std::printf(" %llu", static_cast<unsigned long long>(v.strides[d]));
    for (int d = 0; d < v.rank; ++d) std::printf(" %u", static_cast<unsigned>(v.box[d]));
    std::printf("\n");
}

int main(int argc, char** argv) {
    if (argc != 4) {
        std::fprintf(stderr, "usage: %s E I H\n", argv[0]);
        return 2;
    }
    const int E = std::atoi(argv[1]), I = std::atoi(argv[2]), H = std::atoi(argv[3]);
    View v;
    // the prefill pair kernel (fragment order, 128-row boxes)
    print("pair_fc1_interleaved", moe::tmap::quad_rows_view(&v, E, 2 * I, H), v);
    print("pair_fc1_chunked", moe::tmap::fc1_quad_rows_chunked_view(&v, E, I, H), v);
    print("pair_fc2", moe::tmap::quad_rows_view(&v, E, H, I), v);
    // the decode kernel (pair order, 64-pair boxes), bf16 and int8
    for (int u8 = 0; u8 < 2; ++u8) {
        print(u8 ? "decode_fc1_interleaved_u8" : "decode_fc1_interleaved",
              moe::tmap::fc1_pairs_view(&v, E, I, H, 64, false, u8 != 0), v);
        print(u8 ? "decode_fc1_chunked_u8" : "decode_fc1_chunked",
              moe::tmap::fc1_pairs_view(&v, E, I, H, 64, true, u8 != 0), v);
        print(u8 ? "decode_fc2_u8" : "decode_fc2",
              moe::tmap::plain_pairs_view(&v, E, H, I, 64, u8 != 0), v);
    }
    return 0;
}
