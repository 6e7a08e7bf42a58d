// nf4_table.h -- the NF4 codebook used by every kernel of the library.
//
// "LoRA and QLoRA" (chkda.github.io/posts/lora_qlora), sections "NF4: Choose
// the codebook to fit the distribution" and "Building the NF4 codebook": 16
// reconstruction values from quantiles of N(0, 1), normalised to [-1, 1], with
// an exact zero, seven negative and eight positive values.  The page prints
// the values to four decimals and leaves the quantiles' tail cutoff open.
//
// These are the fp32 values of the construction
//     C = { Phi^-1(1/2 + (p*-1/2) i/8) / Phi^-1(p*), i = 1..8 }
//       u { -Phi^-1(1/2 + (p*-1/2) i/7) / Phi^-1(p*), i = 1..7 } u { 0 }
// with p* = 0.9677053338292209, the midpoint of the interval of cutoffs
// (0.96770238..0.96770828) for which all 16 printed values are reproduced.
// Ascending order; C[7] = 0, C[0] = -1, C[15] = +1.
#pragma once

#define QLORA_NF4_TABLE_BITS                                                                      \
  0xbf800000u, 0xbf323a31u, 0xbf066ba6u, 0xbeca3362u, 0xbe91a2deu, 0xbe3d3601u, 0xbdba792cu,    \
      0x00000000u, 0x3da2fbacu, 0x3e24cb8au, 0x3e7c05dbu, 0x3ead03e2u, 0x3ee1a58au, 0x3f100825u, \
      0x3f39142eu, 0x3f800000u

#define QLORA_NF4_ZERO_CODE 7
