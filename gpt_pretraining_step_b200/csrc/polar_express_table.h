// Newton-Schulz coefficient table of Muon (host side, computed once).
#pragma once

namespace gpt {

constexpr int kPolarSteps = 5;

// (a, b, c) per step, in application order.
const double (*polar_coefficients())[3];

}  // namespace gpt
