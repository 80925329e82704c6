// tc_gdn.cu -- placeholder until the tcgen05 kernel lands.
#include "tc_gdn.h"
namespace hlta {
TcGdn *TcGdn::create(const hlta_config &, long long) { return nullptr; }
}  // namespace hlta
