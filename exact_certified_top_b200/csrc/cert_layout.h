// Layout of the per-query certificate record written by cert_setup and read by
// the certified scorer (and returned to callers by dosa_index_certificate).
#pragma once

namespace dosa {

constexpr int kCertFloats = 16;     // floats per query
constexpr int kCertOmega = 0;       // [4] folded weights of the retained heads
constexpr int kCertBeta = 4;        // coefficient of ||k|| (residuals + slack + split error)
constexpr int kCertMargin = 5;      // c: the candidate margin is c * ||k||
constexpr int kCertScale = 6;       // [4] scales of bound rows 4..7 (u_1 hi, lo, u_2 hi, lo)
constexpr int kCertBetaSum = 10;    // per-head Cauchy-Schwarz sum (report)
constexpr int kCertBetaJoint = 11;  // joint spectral bound (report)
constexpr int kCertNA1 = 12;        // |A_1| (report)
constexpr int kCertNA2 = 13;        // |A_2| (report)
constexpr int kCertNO = 14;         // number of omitted positive heads (report)
constexpr int kBoundRows = 8;       // bound directions per query

}  // namespace dosa
