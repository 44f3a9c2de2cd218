// Fused RPBH linear layer (see rpbh_linear.cu). Internal interface for the fault read-out in
// tq3.cu; the entry point itself, rpbh_linear, is declared in wq.h.
#pragma once

namespace wq {
namespace rpbh_linear {

// Reads and clears the fault bits of the kernel (bit 4: a bounded wait ran out).
unsigned int read_and_clear_fault();

}  // namespace rpbh_linear
}  // namespace wq
