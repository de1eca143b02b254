// Bit layout of one weight plane, shared by the host encoder and the device kernels.
//
// A plane of a matrix with R rows and C columns holds one bit per weight (R*C/8 bytes).
// Words are ordered [R/16 row tiles][C/64 column blocks][32 lanes]. Lane l = 4*g + c of a
// tile/block word covers rows {g, g+8} and 8 columns of each 32-column half of the block, in
// the order the u8 x s8 m16n8k32 MMA expects its A fragments: "nibble m, position rho" of the
// lane is the weight at
//   row    = 16*tile + g + 8*(rho & 1)
//   column = 64*block + 32*(m & 1) + 16*(rho >> 1) + 4*c + (m >> 1)
// (m = 0..7, rho = 0..3): gathering position rho of all B planes gives one register of 8
// 4-bit codes whose even nibbles are the A bytes of the first 32-column MMA and whose odd
// nibbles are (16x) the A bytes of the second.
// Where in the word that weight's bit sits depends on the format:
//   binary-coded planes: bit 4*m + rho;
//   uniform codes:       bit (4*m + (B-1-p) - rho) mod 32 in plane p (code bit B-1-p).
// The uniform placement puts plane p's bits of position rho where the code bit belongs after
// one rotation by rho that is the same for every plane: a decoder merges the planes' words with
// fixed masks and rotates once per rho, instead of shifting every plane into place.
#pragma once
#include <cstdint>

namespace dpa_layout {

struct BitPos {
    uint64_t word;
    int bit;
};

inline BitPos bit_position(int C, int row, int col, int plane, int B, bool uniform) {
    const int tile = row >> 4, rt = row & 15;
    const int g = rt & 7, rho_lo = rt >> 3;
    const int block = col >> 6, cb = col & 63;
    const int m_lo = cb >> 5, rem = cb & 31;
    const int rho_hi = rem >> 4, rem2 = rem & 15;
    const int c = rem2 >> 2, m_hi = rem2 & 3;
    const int rho = rho_lo + 2 * rho_hi, m = m_lo + 2 * m_hi;
    const int lane = 4 * g + c;
    const uint64_t nblocks = static_cast<uint64_t>(C) >> 6;
    BitPos bp;
    bp.word = ((static_cast<uint64_t>(tile) * nblocks + block) << 5) + lane;
    bp.bit = uniform ? ((4 * m + (B - 1 - plane) - rho) & 31) : 4 * m + rho;
    return bp;
}

}  // namespace dpa_layout
