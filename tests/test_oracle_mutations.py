"""Pin sensitivity: plant plausible slips in copies of the oracle (on the CPU)
and check that the pins in test_oracle_pins.py catch every one of them.

A slip that no pin caught would mean the oracle could be wrong in that way
without any test noticing.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

# (name, exact source text, replacement)
MUTATIONS = [
    ("drop n_j weight", "dot * inv_sqrt_d + log((double)nj)", "dot * inv_sqrt_d"),
    ("scale 1/D instead of 1/sqrt(D)", "1.0 / sqrt((double)D)", "1.0 / (double)D"),
    ("entropy sign", "h -= (double)row[j]", "h += (double)row[j]"),
    ("entropy mean over C_k", "H[bh] = acc / Cq;", "H[bh] = acc / Ck;"),
    ("frame-0 last block off by one", "*last = (end - 1) / L->q_block;", "*last = end / L->q_block;"),
    ("frame-0 first block rounded up", "*first = start / L->q_block;",
     "*first = (start + L->q_block - 1) / L->q_block;"),
    ("cut entry excluded", "if (c >= p)", "if (c > p)"),
    ("ties to the higher index", "return (x->j > y->j) - (x->j < y->j);",
     "return (x->j < y->j) - (x->j > y->j);"),
    ("ascending order", "if (x->p > y->p) return -1;", "if (x->p > y->p) return 1;"),
    ("pool divides by block size", "out[r * D + d] = (float)(n > 0 ? s / n : 0.0);",
     "out[r * D + d] = (float)(n > 0 ? s / block : 0.0);"),
    ("text blocks floored", "(L->text_len + L->k_block - 1) / L->k_block", "L->text_len / L->k_block"),
    ("padded keys attended", "int cnt = ora_block_count(L->seq_len, bk, j);", "int cnt = bk;"),
    ("attention scale dropped", "s[a] = dot * scale;", "s[a] = dot;"),
    ("lse without log", "(float)(m + log(z))", "(float)(m + z)"),
    ("text keep on query rows", "for (int j = 0; j < tk; ++j) m[j] = 1;",
     "for (int j = 0; j < tk && i < tk; ++j) m[j] = 1;"),
    ("value norm of the block sum", "double c = n > 0 ? s / n : 0.0;", "double c = s;"),
    ("high-entropy heads pooled", "low[(long)b * nh + o[k].h] = 1;", "low[(long)b * nh + o[nh - 1 - k].h] = 1;"),
    ("pool ranked by P' alone", "return p * v;", "return p;"),
    ("pool target not scaled by the total", "const double target = (double)pool_p * T;",
     "const double target = (double)pool_p;"),
    ("pool cut entry excluded", "if (c >= target)", "if (c > target)"),
    ("pool ties by descending row", "if (x->i != y->i) return (x->i > y->i) - (x->i < y->i);",
     "if (x->i != y->i) return (x->i < y->i) - (x->i > y->i);"),
    ("no safeguard", "m[best] = 1;", "(void)best;"),
    ("safeguard takes the last maximum", "if (x > bv) { bv = x; best = j; }",
     "if (x >= bv) { bv = x; best = j; }"),
    ("weight pi instead of 1 / pi", "w[e] = p > 0.0f ? 1.0f / p : 0.0f;", "w[e] = p > 0.0f ? p : 0.0f;"),
    ("sum of exp terms not reweighted", "z += e;",
     "z += e / (weight ? (double)weight[r * Ck + u_of[a] / bk] : 1.0);"),
    ("inclusion probability not capped at one", "float p = prod < 1.0f ? prod : 1.0f;", "float p = prod;"),
    ("overrides sampled like the rest", "if (forced[e]) p = 1.0f;", "(void)forced;"),
    ("draw ignores the seed", "uint64_t z = seed + (idx + 1u) * 0x9E3779B97F4A7C15ull;",
     "uint64_t z = (idx + 1u) * 0x9E3779B97F4A7C15ull;"),
    ("sub-clusters seeded from the first tokens", "int t0 = n > 0 ? (int)(((long)k * n) / nsub) : 0;",
     "int t0 = n > 0 ? (k < n ? k : n - 1) : 0;"),
    ("sub-cluster rows weighted equally", "const double wk = (double)nk / (double)ntot;",
     "const double wk = 1.0 / (double)nsub;"),
    ("sub-cluster ties to the higher index", "if (dist < bd) { bd = dist; best = k; }",
     "if (dist <= bd) { bd = dist; best = k; }"),
    ("neighbor and current frames swapped", "int grp = f == 0 ? 0 : (f == F - 1 ? 2 : 1);",
     "int grp = f == 0 ? 0 : (f == F - 1 ? 1 : 2);"),
    ("dummy heads by the largest l", "if (ora_dhp_l[x] < ora_dhp_l[y]) return -1;",
     "if (ora_dhp_l[x] < ora_dhp_l[y]) return 1;"),
    ("opportunity cost from the sink alone",
     "l[h] = alpha[h * 3] > alpha[h * 3 + 1] ? alpha[h * 3] : alpha[h * 3 + 1];", "l[h] = alpha[h * 3];"),
    ("grouped domain pools swapped", "case 2: pool_of[r] = low[r] ? 0 : 1; G = 2; break;",
     "case 2: pool_of[r] = low[r] ? 1 : 0; G = 2; break;"),
    ("per-head domain in one pool", "case 1: pool_of[r] = (int8_t)h; G = L->heads; break;",
     "case 1: pool_of[r] = 0; G = L->heads; break;"),
    ("distortion without the row renormalisation", "om = z > 0.0 ? om / z : 0.0;",
     "om = z > 0.0 ? om : 0.0;"),
    ("queries from the first frame", "for (int t = (F - 1) * T; t < F * T; t += query_stride) {",
     "for (int t = 0; t < T; t += query_stride) {"),
]


def _build_variant(src, tmpdir, tag):
    path = os.path.join(tmpdir, "mut_%s.c" % tag)
    with open(path, "w") as f:
        f.write(src)
    lib = os.path.join(tmpdir, "libmut_%s.so" % tag)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                    path, "-o", lib, "-lm"], check=True, capture_output=True)
    return oracle.Oracle(lib)


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_slip(name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, "mutation anchor not unique: %r" % old
    with tempfile.TemporaryDirectory() as d:
        ora = _build_variant(src.replace(old, new), d, "x")
        caught = []
        for check in pins.ALL_CHECKS:
            try:
                check(ora)
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(check.__name__)
        assert caught, "no pin caught the planted slip: " + name
