// Internal declarations shared by the host builders (tq_host.cpp) and the CUDA library (tq_lib.cu).
#pragma once

#include <cstdint>

#include "../../include/tq.h"

namespace tq {

// Record a printf-style message for tq_last_error() and return `status`.
tq_status fail(tq_status status, const char* fmt, ...);
void clear_error();

// count standard normal draws of the seeded generator: SplitMix64 outputs 2p and 2p+1 give draws 2p and 2p+1
// through the Box-Muller transform.
void host_gaussians(uint64_t seed, size_t count, double* out);

// Seeded Haar rotation (row-major d*d doubles): QR of a SplitMix64/Box-Muller Gaussian matrix by
// Householder reflections, Q's columns multiplied by sign(diag R) (zero taken as +1).
void host_rotation(int d, uint64_t seed, double* pi);

// Seeded randomized Walsh-Hadamard rotation (row-major d*d doubles, d a power of two):
// Pi = H diag(s) / sqrt(d), H the Sylvester Hadamard matrix, s_j = -1 if the top bit of SplitMix64(seed)
// output j is set, else +1.
void host_hadamard(int d, uint64_t seed, double* pi);

// Either rotation by kind (TQ_ROT_HAAR / TQ_ROT_HADAMARD); false for an unknown kind.
bool host_rotation_of(int kind, int d, uint64_t seed, double* pi);

// Lloyd-Max levels (ascending, 2^bits) of the sphere-coordinate density for dimension d, fp64.
void host_codebook(int d, int bits, double* levels);

// Distortion d * E[(x - Q(x))^2] of levels c / boundaries t (2^bits and 2^bits-1 entries).
double host_distortion(int d, int bits, const double* c, const double* t);

// binary16 <-> double, round to nearest even.
uint16_t f64_to_f16(double v);
double f16_to_f64(uint16_t h);

}  // namespace tq
