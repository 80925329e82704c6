// tc_attention.cu -- placeholder until the tcgen05 kernel lands.
#include "tc_attention.h"
namespace hlta {
TcAttention *TcAttention::create(const hlta_config &, long long) { return nullptr; }
}  // namespace hlta
