// Host-only check of the tcgen05 attention kernel's descriptor encoders
// against CUTLASS's own bitfield unions (cute/arch/mma_sm100_desc.hpp),
// filled with the same fields.
#include <cstdio>
#include <cute/arch/mma_sm100_desc.hpp>
#include "attend_tc.cuh"

int main() {
  int bad = 0;
  for (uint32_t start : {0x0000u, 0x1000u, 0x8420u, 0x3ff90u}) {
    for (uint32_t lbo : {16u, 8192u}) {
      cute::UMMA::SmemDescriptor d;
      d.desc_ = 0;
      d.start_address_ = static_cast<uint16_t>(start >> 4);
      d.leading_byte_offset_ = static_cast<uint16_t>(lbo >> 4);
      d.stride_byte_offset_ = static_cast<uint16_t>(1024 >> 4);
      d.version_ = 1;
      d.base_offset_ = 0;
      d.lbo_mode_ = 0;
      d.layout_type_ = static_cast<uint8_t>(cute::UMMA::LayoutType::SWIZZLE_128B);
      const uint64_t ours = pa::umma_sdesc_sw128(start, lbo, 1024);
      if (uint64_t(d) != ours) { ++bad; printf("smem desc start=%x lbo=%u cutlass=%016llx ours=%016llx\n", start, lbo, (unsigned long long)uint64_t(d), (unsigned long long)ours); }
    }
  }
  struct { int m, n; bool amn, bmn; } shapes[] = {{128, 64, false, false}, {128, 128, false, true}, {64, 32, true, false}};
  for (auto s : shapes) {
    cute::UMMA::InstrDescriptor i;
    i.desc_ = 0;
    i.c_format_ = 1;   // F32
    i.a_format_ = 1;   // BF16
    i.b_format_ = 1;   // BF16
    i.a_major_ = s.amn ? 1 : 0;
    i.b_major_ = s.bmn ? 1 : 0;
    i.n_dim_ = s.n >> 3;
    i.m_dim_ = s.m >> 4;
    const uint32_t ours = pa::umma_idesc_bf16(s.m, s.n, s.amn, s.bmn);
    if (uint32_t(i) != ours) { ++bad; printf("instr desc m=%d n=%d cutlass=%08x ours=%08x\n", s.m, s.n, uint32_t(i), ours); }
  }
  printf("descriptors: %s\n", bad ? "MISMATCH" : "equal to CUTLASS's bitfields");
  return bad ? 1 : 0;
}
