// repack.cu -- canonical NVFP4 weights -> the tiled layout the expert kernels read.
//
// Tile (128 rows x 64 reduction elements) of projection matrix M of expert e:
//   codes  : 4096 bytes = [half h of the 64 columns][row r of 128][16 bytes]
//            byte b of (h, r) holds columns 32h + 2b (low nibble) and 32h + 2b + 1
// Tiles are stored [expert][row tile][column tile], so a row tile's columns
// are contiguous. The scales of a tile form one 512-byte slab stored in the
// same order: [128 rows][4 scale bytes of the row's 4 16-column blocks].
// Gate and up share one matrix of 2I rows: row 2j is gate row j and row 2j+1
// is up row j.
#include "common.cuh"
#include "internal.h"

namespace tfmoe {
namespace {

// One thread per (expert, tiled row, column tile): copies 2 x 16 code bytes and 4 scale bytes.
// Source row r of expert e starts at element (e * rows + r) * K; with split_ld > 0 the source
// is one matrix of rows of split_ld elements whose column block [e*K, (e+1)*K) is expert e
// (the shared expert's down projection, cut along its reduction dimension into slots).
__global__ void repack_kernel(const uint8_t *__restrict__ codes_a, const uint8_t *__restrict__ scales_a,
                              const uint8_t *__restrict__ codes_b, const uint8_t *__restrict__ scales_b,
                              int E, int R, int K, uint8_t *__restrict__ out_codes, uint8_t *__restrict__ out_scales,
                              int split_ld = 0)
{
    // interleaved (codes_b != nullptr): tiled row r -> source (r & 1 ? b : a) row r >> 1
    const int KT = K / kTileK, RT = R / kTileRows;
    const size_t n = (size_t)E * R * KT;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int kt = (int)(i % KT);
        const int r = (int)((i / KT) % R);
        const int e = (int)(i / ((size_t)KT * R));
        const uint8_t *sc, *sr;
        int src_row, src_rows;
        if (codes_b) {
            src_row = r >> 1;
            src_rows = R / 2;
            sc = (r & 1) ? codes_b : codes_a;
            sr = (r & 1) ? scales_b : scales_a;
        } else {
            src_row = r;
            src_rows = R;
            sc = codes_a;
            sr = scales_a;
        }
        const size_t elem = split_ld > 0 ? (size_t)src_row * split_ld + (size_t)e * K
                                         : ((size_t)e * src_rows + src_row) * K;
        const uint8_t *crow = sc + elem / 2 + (size_t)kt * 32;
        const uint8_t *srow = sr + elem / 16 + (size_t)kt * 4;
        const size_t tile = ((size_t)e * RT + r / kTileRows) * KT + kt;
        uint8_t *ct = out_codes + tile * kTileCodeBytes + (r % kTileRows) * 16;
        *reinterpret_cast<uint4 *>(ct) = *reinterpret_cast<const uint4 *>(crow);
        *reinterpret_cast<uint4 *>(ct + 2048) = *reinterpret_cast<const uint4 *>(crow + 16);
        const size_t rti = (size_t)e * RT + r / kTileRows;
        *reinterpret_cast<uint32_t *>(out_scales + scale_offset(rti, KT, kt) + (r % kTileRows) * 4) =
            *reinterpret_cast<const uint32_t *>(srow);
    }
}

}  // namespace

cudaError_t launch_repack(const Layer &L, const tfmoe_weights &src, cudaStream_t s)
{
    const int H = L.desc.hidden, I = L.desc.intermediate, E = L.desc.num_experts;
    repack_kernel<<<4 * L.num_sms, 256, 0, s>>>(src.gate_codes, src.gate_scales, src.up_codes, src.up_scales,
                                                 E, 2 * I, H, L.w.gu_codes, L.w.gu_scales);
    repack_kernel<<<4 * L.num_sms, 256, 0, s>>>(src.down_codes, src.down_scales, nullptr, nullptr,
                                                 E, H, I, L.w.d_codes, L.w.d_scales);
    const int m = shared_slots(L);
    if (m > 0) {
        // the shared expert's m slots follow the routed experts: gate/up rows [m][I] as m
        // experts, the down projection's columns cut into m blocks of I
        const size_t gu_tiles = (size_t)E * (2 * I / kTileRows) * (H / kTileK);
        const size_t d_tiles = (size_t)E * (H / kTileRows) * (I / kTileK);
        repack_kernel<<<4 * L.num_sms, 256, 0, s>>>(src.shared_gate_codes, src.shared_gate_scales,
                                                     src.shared_up_codes, src.shared_up_scales, m, 2 * I, H,
                                                     L.w.gu_codes + gu_tiles * kTileCodeBytes,
                                                     L.w.gu_scales + gu_tiles * kTileScaleBytes);
        repack_kernel<<<4 * L.num_sms, 256, 0, s>>>(src.shared_down_codes, src.shared_down_scales, nullptr, nullptr,
                                                     m, H, I, L.w.d_codes + d_tiles * kTileCodeBytes,
                                                     L.w.d_scales + d_tiles * kTileScaleBytes, m * I);
    }
    return cudaGetLastError();
}

}  // namespace tfmoe
