// MXFP4 weight packer: canonical layout <-> streaming device layout.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) traces a wrong-but-fast path to
// a W2 layout mismatch that permuted expert outputs, and repairs the layout at
// load time.  Here the device layout is produced once by moe_pack_weights and
// is checked by the exact inverse, moe_unpack_weights, whose output must
// reproduce the canonical bytes.
//
// Device layout (one layout serves both the CUDA-core streaming GEMM and the
// tensor-core GEMM).  Per expert, W1 region then W2 region; one expert matrix
// with N rows and K inputs is split into 128-row blocks rb and 128-input
// groups g, chunk (rb, g) at byte offset (rb * K/128 + g) * 8704:
//   [   0,  512)  scales: byte l*16 + t*4 + j = UE8M0 scale of device row
//                 rb*128 + t*32 + l, input block 4g + j (l < 32, t < 4, j < 4);
//                 the tensor cores' 128-row x 4-block scale-factor atom
//   [ 512, 8704)  codes:  16 bytes at 512 + j*2048 + t*512 + l*16 = the 32 E2M1
//                 codes (canonical nibble order) of that row and block; i.e. for
//                 every block j the 128 rows' 16-byte pieces back to back, the
//                 no-swizzle K-major core-matrix order of the tensor cores
// A warp of the streaming GEMM (lane l = rows l of two adjacent 32-row tiles t,
// t + 1) reads two adjacent 512-byte slices, 1 KB contiguous, per block; the
// tensor-core producer fetches a whole chunk with one bulk copy.
// Device rows of W2 are its canonical rows.  Device rows of W1 interleave gate
// and up rows per 32-row tile: device row 32*tau + r is gate row 16*tau + r
// for r < 16 and up row I + 16*tau + (r - 16) otherwise, so every warp-sized
// group of rows holds the gate and up rows of the same 16 outputs.
// The layout moves the canonical bytes, so its size equals the canonical size.
#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {


__host__ __device__ inline size_t matrix_bytes(int N, int K) { return (size_t)N * K * 17 / 32; }

// byte offsets, inside one expert matrix, of the scale byte / first code byte of
// (device row d, input block b)
__host__ __device__ inline size_t dl_scale_off(int d, int b, int K) {
    const int rb = d >> 7, t = (d >> 5) & 3, l = d & 31, g = b >> 2, j = b & 3;
    return ((size_t)rb * (K / 128) + g) * 8704 + l * 16 + t * 4 + j;
}
__host__ __device__ inline size_t dl_code_off(int d, int b, int K) {
    const int rb = d >> 7, t = (d >> 5) & 3, l = d & 31, g = b >> 2, j = b & 3;
    return ((size_t)rb * (K / 128) + g) * 8704 + 512 + j * 2048 + t * 512 + l * 16;
}

// One thread per (expert, device row, 32-element block).  forward: canonical ->
// device.  gate_up_half > 0 selects the W1 row interleave with that I.
template <bool kForward>
__global__ void k_pack_matrix(uint8_t* __restrict__ dev, uint8_t* __restrict__ codes,
                              uint8_t* __restrict__ scales, int E, int N, int K, int gate_up_half,
                              int32_t* flag) {
    const int nb = K / 32;
    const size_t total = (size_t)E * N * nb;
    const size_t mbytes = matrix_bytes(N, K);
    bool bad = false;
    for (size_t id = blockIdx.x * (size_t)blockDim.x + threadIdx.x; id < total;
         id += (size_t)gridDim.x * blockDim.x) {
        const int b = (int)(id % nb);
        const size_t rd = id / nb;
        const int drow = (int)(rd % N);
        const int e = (int)(rd / N);
        int crow = drow;  // canonical row of this device row
        if (gate_up_half > 0) {
            const int tau = drow >> 5, r = drow & 31;
            crow = (r < 16) ? tau * 16 + r : gate_up_half + tau * 16 + (r - 16);
        }
        const size_t rn = (size_t)e * N + crow;
        uint8_t* d = dev + (size_t)e * mbytes;
        uint4* cc = reinterpret_cast<uint4*>(codes + rn * (K / 2) + (size_t)b * 16);
        uint8_t* cs = scales + rn * nb + b;
        uint4* dc = reinterpret_cast<uint4*>(d + dl_code_off(drow, b, K));
        uint8_t* ds = d + dl_scale_off(drow, b, K);
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
                                                          E, 2 * I, H, I, &hdr->flag);
        count_launches(1);
        k_pack_matrix<true><<<grid_for(n2), 256, 0, st>>>(base + L.w2, (uint8_t*)w2c, (uint8_t*)w2s,
                                                          E, H, I, 0, &hdr->flag);
        count_launches(1);
    } else {
        const size_t n1 = (size_t)E * 2 * I * (H / 32), n2 = (size_t)E * H * (I / 32);
        k_pack_matrix<false><<<grid_for(n1), 256, 0, st>>>(base + L.w1, out_w1c, out_w1s, E, 2 * I,
                                                           H, I, nullptr);
        count_launches(1);
        k_pack_matrix<false><<<grid_for(n2), 256, 0, st>>>(base + L.w2, out_w2c, out_w2s, E, H, I,
                                                           0, nullptr);
        count_launches(1);
    }
    return cudaGetLastError();
}

const int32_t* packed_flag_ptr(const void* packed) {
    return &((const PackHeader*)packed)->flag;
}


}  // namespace moe
