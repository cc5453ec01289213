"""The oracle pins must catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake there (a flipped sign, a wrong index or head mapping, a dropped term,
a wrong position), compiles it and runs the pin suite against the broken
library in a child process; the pins must fail.  Nothing is planted in the
committed oracle.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "msa_oracle.c")

MUTANTS = {
    "rope_sign": ("y[i] = x0 * c - x1 * s;", "y[i] = x0 * c + x1 * s;"),
    "rope_exponent": ("-2.0 * (double)i / (double)d", "-1.0 * (double)i / (double)d"),
    "rope_pairing": ("double x0 = x[i], x1 = x[i + h];", "double x0 = x[i], x1 = x[h - 1 - i];"),
    "encode_no_position_reset": ("rope_w(x, d, (double)p, w, y);", "rope_w(x, d, (double)(t0 + p), w, y);"),
    "encode_divides_by_chunk": ("k_pool[(c * H + g) * (int64_t)d + i] = acc[i] / (double)n;",
                                "k_pool[(c * H + g) * (int64_t)d + i] = acc[i] / (double)chunk;"),
    "route_head_mapping": ("int g = h / G;", "int g = h % Hkv;"),
    "route_no_head_mean": ("double S = sum / (double)Hq;", "double S = sum;"),
    "route_kr_norm_squared": ("kn[g] = sqrt(nn);", "kn[g] = nn;"),
    "route_tie_break": ("if (arg < 0 || score[s] > score[arg]) arg = s;  /* strict",
                        "if (arg < 0 || score[s] >= score[arg]) arg = s;  /* strict"),
    "interleave_reselects": ("if (taken[s]) continue;\n        if (arg < 0 || score[s] > score[arg]) arg = s;\n      }\n      taken[arg] = 1;\n      sel_new",
                             "if (0) continue;\n        if (arg < 0 || score[s] > score[arg]) arg = s;\n      }\n      taken[arg] = 1;\n      sel_new"),
    "interleave_tie_break": ("if (arg < 0 || score[s] > score[arg]) arg = s;\n      }\n      taken[arg] = 1;\n      sel_new",
                             "if (arg < 0 || score[s] >= score[arg]) arg = s;\n      }\n      taken[arg] = 1;\n      sel_new"),
    "decode_no_global_offset": ("rope_w(qv, d, (double)(top_k + Lb + t), w, qrot);",
                                "rope_w(qv, d, (double)(Lb + t), w, qrot);"),
    "decode_no_scale": ("logit[j] = dot / scale_div;", "logit[j] = dot;"),
    "decode_not_causal": ("int64_t visible = nmem + Lb + t + 1;", "int64_t visible = nmem + Ltot;"),
    "decode_keys_as_values": ("vals[n * d + i] = ld(vsrc, dtype, (vrow * Hkv + g) * (int64_t)d + i);",
                              "vals[n * d + i] = ld(k_pool, dtype, (krow * Hkv + g) * (int64_t)d + i);"),
    "bf16_shift": ("uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;",
                   "uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 15;"),
    "bf16_byte_order": ("uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;",
                        "uint32_t u = (uint32_t)__builtin_bswap16(((const uint16_t*)p)[i]) << 16;"),
    "decode_local_keys_unrotated": ("rope_w(x, d, (double)(top_k + j), w, keys + n * d);",
                                    "memcpy(keys + n * d, x, sizeof(double) * (size_t)d);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mut = tmp_path / "msa_oracle.c"
    mut.write_text(src.replace(old, new))
    (tmp_path / "msa_oracle.h").write_text(open(os.path.join(ROOT, "oracle", "msa_oracle.h")).read())
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(so), str(mut), "-lm"], check=True)
    env = dict(os.environ, MSA_ORACLE_LIB=str(so), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
