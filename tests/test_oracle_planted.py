"""Plant one plausible mistake at a time in a copy of the oracle's C source and check
that at least one pin catches it: the pins are not blind to dropped terms, wrong
signs or indices, or transposed operands."""
import os

import pytest

import oracle
import oracle_pins

# (name, exact text in oracle.c, replacement)
PLANTS = [
    ("scale dropped from the scores", "s *= scale;", "s *= 1.0;"),
    ("window bound off by one", "if (left >= 0 && j < i - left) return 0;",
     "if (left >= 0 && j <= i - left) return 0;"),
    ("causal flag ignored", "if (right < 0 || right > 0) return 0;", "if (0) return 0;"),
    ("row maximum left out of LSE", "lse[i] = m + log(sum);", "lse[i] = log(sum);"),
    ("softmax not normalised", "for (j = 0; j < N; ++j) Pi[j] /= sum;",
     "for (j = 0; j < N; ++j) Pi[j] /= 1.0;"),
    ("O row index swapped", "oh[i * d + c] += p * vh[j * d + c];",
     "oh[i * d + c] += p * vh[i * d + c];"),
    ("dV uses P instead of P^T", "double p = Pd[ii * N + j];", "double p = Pd[j * N + ii];"),
    ("dS sign of D flipped", "(dP[i * N + jj] - D[i])", "(dP[i * N + jj] + D[i])"),
    ("dQ scale dropped", "dqh[i * d + c] *= scale;", "dqh[i * d + c] *= 1.0;"),
    ("dK uses dS instead of dS^T", "double s = dP[ii * N + j];", "double s = dP[j * N + ii];"),
    ("dK scale dropped", "dkh[j * d + c] *= scale;", "dkh[j * d + c] *= 1.0;"),
    ("dP uses dO of the key row", "s += doh[i * d + c] * vh[jj * d + c];",
     "s += doh[jj * d + c] * vh[jj * d + c];"),
    ("ALiBi bias sign flipped", "s += -slope * fabs((double)(i - j));",
     "s += slope * fabs((double)(i - j));"),
    ("ALiBi distance without the absolute value", "s += -slope * fabs((double)(i - j));",
     "s += -slope * (double)(i - j);"),
    ("ALiBi bias scaled with the scores", "s += -slope * fabs((double)(i - j));",
     "s += -slope * scale * fabs((double)(i - j));"),
    ("ALiBi slope of the wrong head", "return alibi_slopes ? alibi_slopes[bh % H] : 0.0;",
     "return alibi_slopes ? alibi_slopes[0] : 0.0;"),
    ("key padding ignored", "if (kpad && kpad[j]) s = -INFINITY;", "if (0) s = -INFINITY;"),
    ("key padding applied by query", "if (kpad && kpad[j]) s = -INFINITY;",
     "if (kpad && kpad[i]) s = -INFINITY;"),
    ("key padding of the first batch entry for all",
     "return key_padding ? key_padding + (bh / H) * N : NULL;",
     "return key_padding ? key_padding : NULL;"),
    ("lengths applied to keys only", "if (i >= len || j >= len) s = -INFINITY;",
     "if (j >= len) s = -INFINITY;"),
    ("lengths of the first entry for all", "return lengths ? lengths[bh / H] : N;",
     "return lengths ? lengths[0] : N;"),
    ("Philox multiplier typo", "M0 = 0xD2511F53u", "M0 = 0xD2511F55u"),
    ("Philox key not bumped", "k1 += W1;", "k1 += 0;"),
    ("dropout counter takes the key as row", "ctr[1] = (uint32_t)i;", "ctr[1] = (uint32_t)j;"),
    ("dropout threshold off by one", "return (int)byte >= t ? 1 : 0;",
     "return (int)byte > t ? 1 : 0;"),
    ("dropout kept weights not rescaled",
     "P[i * N + j] = dropout_keep(seed, offset, bh, i, j, t) ? P[i * N + j] * keep_scale : 0.0;",
     "P[i * N + j] = dropout_keep(seed, offset, bh, i, j, t) ? P[i * N + j] : 0.0;"),
    ("dropout flags left out of dP", "dP[i * N + jj] = s * zs;", "dP[i * N + jj] = s;"),
]


@pytest.mark.parametrize("name,old,new", PLANTS, ids=[p[0] for p in PLANTS])
def test_plant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, "plant site must be unique: %r" % old
    bad = tmp_path / "oracle_planted.c"
    bad.write_text(src.replace(old, new))
    lib = oracle.build(str(bad), str(tmp_path / "liboracle_planted.so"), force=True)
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, "no pin catches the planted mistake: %s" % name
