"""Plants plausible mistakes in scratch copies of the oracle (on the CPU) and
checks that the pins catch every one of them.

Each mutant is a one-line textual change to ``oracle/mmf_oracle.c``, compiled
into a temporary directory; the real oracle is never touched.
"""
import os

import pytest

import pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mmf_oracle.c")

# (name, text in the source, replacement)
MUTANTS = [
    ("subtract-becomes-add", "else if (wn[k] == -1) s -= qm[k];", "else if (wn[k] == -1) s += qm[k];"),
    ("multiply-by-beta", "const float t = W[i] / d;", "const float t = W[i] * d;"),
    ("round-half-away", "const float r = rintf(t);", "const float r = roundf(t);"),
    ("quant-round-half-away", "const float t = rintf(r * s);", "const float t = roundf(r * s);"),
    ("drop-gamma", "const float r = (orc_bf16_to_f32(xm[k]) * inv) * gamma[k];",
     "const float r = (orc_bf16_to_f32(xm[k]) * inv);"),
    ("max-not-absmax", "const float ar = fabsf(r);", "const float ar = r;"),
    ("sum-not-mean", "const float ms = (float)(s2 / (double)K);", "const float ms = (float)s2;"),
    ("eps-outside-sqrt", "const float inv = 1.0f / sqrtf(ms + eps);",
     "const float inv = 1.0f / (sqrtf(ms) + eps);"),
    ("transposed-acc", "acc[m * N + n] = s;", "acc[n * M + m] = s;"),
    ("natural-bit-order", "const int shift = 8 * (i % 4) + 2 * (i / 4);\n                w |= code << shift;",
     "const int shift = 2 * i;\n                w |= code << shift;"),
    ("qb-128", "const double deq = ((double)absmax[m] / 127.0) * (double)beta;",
     "const double deq = ((double)absmax[m] / 128.0) * (double)beta;"),
    ("drop-beta", "const double deq = ((double)absmax[m] / 127.0) * (double)beta;",
     "const double deq = ((double)absmax[m] / 127.0);"),
    ("beta-plus-eps-sum", "for (int64_t i = 0; i < n; ++i) s += fabs((double)W[i]);",
     "for (int64_t i = 0; i < n; ++i) s += (double)W[i];"),
    ("bf16-truncate", "double s = nearbyint(ldexp(m, 8));", "double s = floor(ldexp(m, 8));"),
    ("code-offset", "const uint32_t code = (uint32_t)(t + 1);", "const uint32_t code = (uint32_t)(t & 3);"),
    ("sigmoid-sign", "const float sig = 1.0f / (1.0f + expf(-gv));", "const float sig = 1.0f / (1.0f + expf(gv));"),
    ("gate-on-u", "const float silu = gv * sig;", "const float silu = uv * sig;"),
    ("forget-swapped", "h = f * h + (1.0f - f) * c;", "h = (1.0f - f) * h + f * c;"),
    ("no-output-gate", "o[i] = orc_f64_to_bf16((double)(g * h));", "o[i] = orc_f64_to_bf16((double)h);"),
    ("silu-as-sigmoid", "const float c = cv * orc_sigmoid(cv);", "const float c = orc_sigmoid(cv);"),
    ("bwd-missing-norm-term", "- xv * inv * inv * inv * dot / (double)K;", "- 0.0 * dot;"),
    ("bwd-dW-unscaled", "((double)q[m * K + k] * ((double)a[m] / 127.0));", "((double)q[m * K + k]);"),
    ("bwd-dr-transposed-w", "s += (double)orc_bf16_to_f32(dy[m * N + n]) * (double)wt[n * K + k];",
     "s += (double)orc_bf16_to_f32(dy[m * N + n]) * (double)wt[(k % N) * K + (n % K)];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    from oracle.build import build
    from oracle.oracle import Oracle

    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    msrc = tmp_path / "mmf_oracle.c"
    msrc.write_text(mutated)
    lib = build(src=str(msrc), out=str(tmp_path / "libmutant.so"), force=True)
    orc = Oracle(lib)
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            failed.append(check.__name__)
        except Exception as e:  # a mutant may also crash a check outright
            failed.append(f"{check.__name__}:{type(e).__name__}")
    assert failed, f"mutant {name} passed every pin"
