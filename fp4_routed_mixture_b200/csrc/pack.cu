// MXFP4 weight packer: canonical layout <-> streaming device layout.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) traces a wrong-but-fast path to
// a W2 layout mismatch that permuted expert outputs, and repairs the layout at
// load time.  Here the device layout is produced once by moe_pack_weights and
// is checked by the exact inverse, moe_unpack_weights, whose output must
// reproduce the canonical bytes.
//
// Streaming device layout of one expert matrix with N rows and K inputs (per
// expert, experts back to back; W1 region then W2 region):
//   tile tau = 32 consecutive rows (row n = 32*tau + lane), tiles back to back;
//   inside a tile, K/128 groups of 4 scale blocks, each 2176 bytes:
//     [  0, 128)  32 lanes x 4 bytes: the lane's UE8M0 scales of blocks 4g..4g+3
//     [128, 640)  32 lanes x 16 bytes: codes of block 4g   (32 nibbles, canonical order)
//     [640,1152)  block 4g+1, [1152,1664) block 4g+2, [1664,2176) block 4g+3
// A warp reading one 512-byte code slice hands each lane one 32-element block
// of its own row, so weight loads are fully coalesced 128-bit loads and no
// cross-lane reduction is needed.  The layout is the canonical bytes moved,
// so its size equals the canonical size.
#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

struct PackHeader {
    uint32_t magic, version, H, I, E, reserved0;
    uint64_t w1_off, w2_off;
    int32_t flag;  // device error word of moe_pack_weights
};

constexpr uint32_t kPackMagic = 0x34454F4Du;  // "MOE4"
constexpr uint32_t kPackVersion = 1;

__host__ __device__ inline size_t matrix_bytes(int N, int K) { return (size_t)N * K * 17 / 32; }

// byte offset, inside one expert matrix, of the scale byte / first code byte of (row n, block b)
__host__ __device__ inline size_t dl_scale_off(int n, int b, int K) {
    const int tau = n >> 5, lane = n & 31, g = b >> 2, bb = b & 3;
    return (size_t)tau * (K / 128) * 2176 + (size_t)g * 2176 + lane * 4 + bb;
}
__host__ __device__ inline size_t dl_code_off(int n, int b, int K) {
    const int tau = n >> 5, lane = n & 31, g = b >> 2, bb = b & 3;
    return (size_t)tau * (K / 128) * 2176 + (size_t)g * 2176 + 128 + bb * 512 + lane * 16;
}

// One thread per (expert, row, 32-element block).  forward: canonical -> device.
template <bool kForward>
__global__ void k_pack_matrix(uint8_t* __restrict__ dev, uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ scales, int E, int N, int K, int32_t* flag) {
    const int nb = K / 32;
    const size_t total = (size_t)E * N * nb;
    const size_t mbytes = matrix_bytes(N, K);
    bool bad = false;
    for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
         id += (size_t)gridDim.x * blockDim.x) {
        const int b = (int)(id % nb);
        const size_t rn = id / nb;
        const int n = (int)(rn % N);
        const int e = (int)(rn / N);
        uint8_t* d = dev + (size_t)e * mbytes;
        uint4* cc = reinterpret_cast<uint4*>(codes + rn * (K / 2) + (size_t)b * 16);
        uint8_t* cs = scales + rn * nb + b;
        uint4* dc = reinterpret_cast<uint4*>(d + dl_code_off(n, b, K));
        uint8_t* ds = d + dl_scale_off(n, b, K);
        if (kForward) {
            const uint8_t s = *cs;
            if (s == 0xFF) bad = true;
            *ds = s;
            *dc = *cc;
        } else {
            *cs = *ds;
            *cc = *dc;
        }
    }
    if (bad) raise_flag(flag, FLAG_BAD_SCALE);
}

__global__ void k_write_header(PackHeader* h, int H, int I, int E, uint64_t w1_off,
                               uint64_t w2_off) {
    h->magic = kPackMagic;
    h->version = kPackVersion;
    h->H = H;
    h->I = I;
    h->E = E;
    h->reserved0 = 0;
    h->w1_off = w1_off;
    h->w2_off = w2_off;
    h->flag = 0;
}

// Raises FLAG_LAYOUT when the packed buffer was built for other dims.
__global__ void k_check_header(const PackHeader* h, int H, int I, int E, int32_t* flag) {
    if (h->magic != kPackMagic || h->version != kPackVersion || (int)h->H != H ||
        (int)h->I != I || (int)h->E != E)
        raise_flag(flag, FLAG_LAYOUT);
}

PackedLayout packed_layout(int H, int I, int E) {
    PackedLayout L;
    L.header = 0;
    L.w1 = 256;
    L.w1_expert_bytes = matrix_bytes(2 * I, H);
    L.w2 = L.w1 + (size_t)E * L.w1_expert_bytes;
    L.w2_expert_bytes = matrix_bytes(H, I);
    L.total = L.w2 + (size_t)E * L.w2_expert_bytes;
    return L;
}

static int grid_for(size_t n) {
    size_t g = (n + 255) / 256;
    return (int)std::min<size_t>(g, 148 * 32);
}

cudaError_t launch_pack(int H, int I, int E, const uint8_t* w1c, const uint8_t* w1s,
                        const uint8_t* w2c, const uint8_t* w2s, void* packed, bool forward,
                        uint8_t* out_w1c, uint8_t* out_w1s, uint8_t* out_w2c, uint8_t* out_w2s,
                        cudaStream_t st) {
    const PackedLayout L = packed_layout(H, I, E);
    uint8_t* base = (uint8_t*)packed;
    PackHeader* hdr = (PackHeader*)(base + L.header);
    if (forward) {
        k_write_header<<<1, 1, 0, st>>>(hdr, H, I, E, L.w1, L.w2);
        count_launches(1);
        const size_t n1 = (size_t)E * 2 * I * (H / 32), n2 = (size_t)E * H * (I / 32);
        k_pack_matrix<true><<<grid_for(n1), 256, 0, st>>>(base + L.w1, (uint8_t*)w1c, (uint8_t*)w1s,
                                                          E, 2 * I, H, &hdr->flag);
        count_launches(1);
        k_pack_matrix<true><<<grid_for(n2), 256, 0, st>>>(base + L.w2, (uint8_t*)w2c, (uint8_t*)w2s,
                                                          E, H, I, &hdr->flag);
        count_launches(1);
    } else {
        const size_t n1 = (size_t)E * 2 * I * (H / 32), n2 = (size_t)E * H * (I / 32);
        k_pack_matrix<false><<<grid_for(n1), 256, 0, st>>>(base + L.w1, out_w1c, out_w1s, E, 2 * I,
                                                           H, nullptr);
        count_launches(1);
        k_pack_matrix<false><<<grid_for(n2), 256, 0, st>>>(base + L.w2, out_w2c, out_w2s, E, H, I,
                                                           nullptr);
        count_launches(1);
    }
    return cudaGetLastError();
}

const int32_t* packed_flag_ptr(const void* packed) {
    return &((const PackHeader*)packed)->flag;
}

cudaError_t launch_check_header(const void* packed, int H, int I, int E, int32_t* flag,
                                cudaStream_t st) {
    k_check_header<<<1, 1, 0, st>>>((const PackHeader*)packed, H, I, E, flag);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
