// NF-k level tables, derived on the host from the inverse normal CDF.
//
// The levels follow the quantile construction of the NF data type (QLoRA explainer,
// "Innovation 1: 4-bit NormalFloat (NF4)": each of the 2^k bins holds an equal share of a
// normal distribution; the values are normalised into [-1, 1]):
//   2^(k-1) positive levels  Phi^-1(p) at p_i = delta + i (1/2 - delta) / 2^(k-1),  i < 2^(k-1)
//   2^(k-1)-1 negative levels -Phi^-1(p) at p_i = delta + i (1/2 - delta) / (2^(k-1) - 1)
//   one exact zero; everything divided by Phi^-1(delta);
//   delta = 1 - (1 / (2 (2^k - 1)) + 1 / (2 * 2^k)) / 2.
// Phi^-1 is Wichura's algorithm AS 241 (PPND16, Applied Statistics 37(3), 1988), a rational
// approximation with about 16 significant digits, evaluated in double precision.  The fp32
// table is the round-to-nearest of each double level.
#include <algorithm>
#include <cmath>
#include <vector>

namespace qlr {

static double poly7(const double* c, double x) {
  double v = c[7];
  for (int i = 6; i >= 0; --i) v = v * x + c[i];
  return v;
}

double normal_quantile(double p) {
  static const double a[8] = {3.3871328727963666080e0, 1.3314166789178437745e+2, 1.9715909503065514427e+3,
                              1.3731693765509461125e+4, 4.5921953931549871457e+4, 6.7265770927008700853e+4,
                              3.3430575583588128105e+4, 2.5090809287301226727e+3};
  static const double b[8] = {1.0, 4.2313330701600911252e+1, 6.8718700749205790830e+2, 5.3941960214247511077e+3,
                              2.1213794301586595867e+4, 3.9307895800092710610e+4, 2.8729085735721942674e+4,
                              5.2264952788528545610e+3};
  static const double c[8] = {1.42343711074968357734e0, 4.63033784615654529590e0, 5.76949722146069140550e0,
                              3.64784832476320460504e0, 1.27045825245236838258e0, 2.41780725177450611770e-1,
                              2.27238449892691845833e-2, 7.74545014278341407640e-4};
  static const double d[8] = {1.0, 2.05319162663775882187e0, 1.67638483018380384940e0, 6.89767334985100004550e-1,
                              1.48103976427480074590e-1, 1.51986665636164571966e-2, 5.47593808499534494600e-4,
                              1.05075007164441684324e-9};
  static const double e[8] = {6.65790464350110377720e0, 5.46378491116411436990e0, 1.78482653991729133580e0,
                              2.96560571828504891230e-1, 2.65321895265761230930e-2, 1.24266094738807843860e-3,
                              2.71155556874348757815e-5, 2.01033439929228813265e-7};
  static const double f[8] = {1.0, 5.99832206555887937690e-1, 1.36929880922735805310e-1, 1.48753612908506148525e-2,
                              7.86869131145613259100e-4, 1.84631831751005468180e-5, 1.42151175831644588870e-7,
                              2.04426310338993978564e-15};
  const double q = p - 0.5;
  if (std::fabs(q) <= 0.425) {
    const double r = 0.180625 - q * q;
    return q * poly7(a, r) / poly7(b, r);
  }
  double r = (q < 0) ? p : 1.0 - p;
  r = std::sqrt(-std::log(r));
  double v;
  if (r <= 5.0) {
    r -= 1.6;
    v = poly7(c, r) / poly7(d, r);
  } else {
    r -= 5.0;
    v = poly7(e, r) / poly7(f, r);
  }
  return (q < 0) ? -v : v;
}

// Fills `out` with the 2^k fp32 levels in ascending order.
void nf_levels_f32(int k, float* out) {
  const int n = 1 << k;
  const int half = n / 2;
  const double delta = 1.0 - 0.5 * (1.0 / (2.0 * (n - 1)) + 1.0 / (2.0 * n));
  std::vector<double> lv;
  const double step_pos = (0.5 - delta) / half;
  for (int i = 0; i < half; ++i) lv.push_back(normal_quantile(delta + i * step_pos));
  if (half > 1) {
    const double step_neg = (0.5 - delta) / (half - 1);
    for (int i = 0; i < half - 1; ++i) lv.push_back(-normal_quantile(delta + i * step_neg));
  }
  lv.push_back(0.0);
  std::sort(lv.begin(), lv.end());
  const double z = normal_quantile(delta);
  for (int i = 0; i < n; ++i) out[i] = static_cast<float>(lv[i] / z);
}

}  // namespace qlr
