"""The oracle's pins catch plausible mistakes (no GPU needed).

Each case plants one slip in a copy of the oracle's C source: a wrong code
order, mask or codes-per-word count, an 8-bit code read as signed, a group size
fixed at 64, a dropped or mis-signed term, a wrong group or row index of a scale
or bias, a transposed operand or router, a missing normalisation or a mean over
H - 1, a reversed tie-break, swapped SwiGLU operands or a sigmoid in place of
SiLU, renormalisation over the wrong probabilities, a missing residual or shared
term; in the Gated DeltaNet step a skipped decay or one applied after the
update, a recall from the undecayed state, a wrong delta sign or a missing delta
term, a dropped or misplaced write strength, a transposed rank-1 update, a
read-out with the wrong vector or before the update.  The copy
is compiled with the oracle's own flags into a temporary directory, the pin suite
(test_oracle_pins.py) runs against it in a child process, and at least one pin
must fail.  The real oracle is never touched.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "fmoe_oracle.c")

# (name, text in the oracle source, the slip that replaces it)
MUTATIONS = [
    ("code order msb-first",
     "return (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);",
     "return (w >> (32 - bits * (1 + c % per_word))) & ((1u << bits) - 1u);"),
    ("bias dropped",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]);"),
    ("bias sign",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) - or_bf16(m->bias[(int64_t)r * gpr + g]);"),
    ("group index of the first group only",
     "const int g = c / m->group;",
     "const int g = 0 * (c / m->group);"),
    ("group size fixed at 64",
     "const int g = c / m->group;",
     "const int g = c / 64;"),
    ("group index by column modulo",
     "const int g = c / m->group;",
     "const int g = c % gpr;"),
    ("matvec transposed",
     "for (int c = 0; c < m->cols; ++c) acc += or_weight(m, r, c) * x[c];",
     "for (int c = 0; c < m->cols; ++c) acc += or_weight(m, c % m->rows, r % m->cols) * x[c];"),
    ("rmsnorm without the mean",
     "const double denom = sqrt(ss / (double)H + eps);",
     "const double denom = sqrt(ss + eps);"),
    ("rmsnorm ignores gamma",
     "x[i] = (double)h[i] / denom * (gamma ? (double)gamma[i] : 1.0);",
     "x[i] = (double)h[i] / denom;"),
    ("router bias dropped",
     "logits[e] = acc + (bias ? (double)bias[e] : 0.0);",
     "logits[e] = acc;"),
    ("softmax not normalised",
     "for (int i = 0; i < n; ++i) p[i] /= s;",
     "for (int i = 0; i < n; ++i) p[i] /= 1.0;"),
    ("top-k ties to the higher index",
     "return (x->i > y->i) - (x->i < y->i);",
     "return (x->i < y->i) - (x->i > y->i);"),
    ("top-k ascending",
     "if (x->v > y->v) return -1;\n  if (x->v < y->v) return 1;",
     "if (x->v > y->v) return 1;\n  if (x->v < y->v) return -1;"),
    ("swiglu operands swapped",
     "g[r] = g[r] / (1.0 + exp(-g[r])) * u[r];",
     "g[r] = u[r] / (1.0 + exp(-u[r])) * g[r];"),
    ("silu sign",
     "g[r] = g[r] / (1.0 + exp(-g[r])) * u[r];",
     "g[r] = g[r] / (1.0 + exp(g[r])) * u[r];"),
    ("weights not renormalised",
     "const double wk = p[idx[k]] / psum;",
     "const double wk = p[idx[k]];"),
    ("shared gate sign",
     "const double sigma = 1.0 / (1.0 + exp(-zs));",
     "const double sigma = 1.0 / (1.0 + exp(zs));"),
    ("shared gate on h instead of the normalised x",
     "for (int i = 0; i < H; ++i) zs += or_bf16(L->w_shared_gate[i]) * x[i];",
     "for (int i = 0; i < H; ++i) zs += or_bf16(L->w_shared_gate[i]) * (double)ht[i];"),
    ("down fed the up projection",
     "or_matvec(&md, g, y);",
     "or_matvec(&md, u, y);"),
    ("eps outside the root",
     "const double denom = sqrt(ss / (double)H + eps);",
     "const double denom = sqrt(ss / (double)H) + eps;"),
    ("gate and up matrices swapped",
     "m.qw = (const uint32_t*)(rec + b->off[3 * which]);\n  m.scale = (const uint16_t*)(rec + b->off[3 * which + 1]);\n"
     "  m.bias = (const uint16_t*)(rec + b->off[3 * which + 2]);",
     "const int wh = which == 2 ? 2 : 1 - which;\n  m.qw = (const uint32_t*)(rec + b->off[3 * wh]);\n"
     "  m.scale = (const uint16_t*)(rec + b->off[3 * wh + 1]);\n  m.bias = (const uint16_t*)(rec + b->off[3 * wh + 2]);"),
    ("scales and biases of a matrix swapped",
     "m.scale = (const uint16_t*)(rec + b->off[3 * which + 1]);\n  m.bias = (const uint16_t*)(rec + b->off[3 * which + 2]);",
     "m.scale = (const uint16_t*)(rec + b->off[3 * which + 2]);\n  m.bias = (const uint16_t*)(rec + b->off[3 * which + 1]);"),
    ("expert record of the next expert",
     "const uint8_t* rec = b->records ? b->records[e] : b->base + (int64_t)e * b->stride;",
     "const uint8_t* rec = b->records ? b->records[(e + 1) % b->num_experts] : b->base + (int64_t)((e + 1) % b->num_experts) * b->stride;"),
    ("residual dropped",
     "for (int i = 0; i < H; ++i) ot[i] = (double)ht[i];",
     "for (int i = 0; i < H; ++i) ot[i] = 0.0;"),
    ("shared expert dropped",
     "for (int i = 0; i < H; ++i) ot[i] += sigma * y[i];",
     "for (int i = 0; i < H; ++i) ot[i] += 0.0 * sigma * y[i];"),
    ("rmsnorm mean over H - 1",
     "const double denom = sqrt(ss / (double)H + eps);",
     "const double denom = sqrt(ss / (double)(H - 1) + eps);"),
    ("scale of the next row",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);",
     "return (double)q * or_bf16(m->scale[(int64_t)((r + 1) % m->rows) * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);"),
    ("bias of the next group",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);",
     "return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + (g + 1) % gpr]);"),
    ("code mask fixed at four bits",
     "return (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);",
     "return (w >> (bits * (c % per_word))) & 0xFu;"),
    ("codes per word fixed at eight",
     "const int per_word = 32 / bits;",
     "const int per_word = 8 + 0 * bits;"),
    ("router transposed",
     "for (int i = 0; i < H; ++i) acc += or_bf16(wr[(int64_t)e * H + i]) * x[i];",
     "for (int i = 0; i < H; ++i) acc += or_bf16(wr[((int64_t)i * E + e) % ((int64_t)E * H)]) * x[i];"),
    ("sigmoid in place of silu",
     "g[r] = g[r] / (1.0 + exp(-g[r])) * u[r];",
     "g[r] = 1.0 / (1.0 + exp(-g[r])) * u[r];"),
    ("renormalised over the first K probabilities",
     "for (int k = 0; k < K; ++k) psum += p[idx[k]];",
     "for (int k = 0; k < K; ++k) psum += p[k];"),
    ("8-bit code read as signed",
     "return (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);",
     "return bits == 8 ? (unsigned)(int)(signed char)((w >> (bits * (c % per_word))) & 0xFFu) : (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);"),
    ("gdn decay skipped",
     "for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] *= a;",
     "for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] *= 1.0;"),
    ("gdn recall from the undecayed state",
     "for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * kh[j];",
     "for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] / a * kh[j];"),
    ("gdn delta sign",
     "Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];",
     "Sh[(int64_t)i * dk + j] += b * (u[i] - vh[i]) * kh[j];"),
    ("gdn no delta term (plain linear attention)",
     "Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];",
     "Sh[(int64_t)i * dk + j] += b * vh[i] * kh[j];"),
    ("gdn write strength dropped",
     "Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];",
     "Sh[(int64_t)i * dk + j] += (vh[i] - u[i]) * kh[j];"),
    ("gdn outer product transposed",
     "Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];",
     "Sh[(int64_t)i * dk + j] += b * (vh[j % dv] - u[j % dv]) * kh[i % dk];"),
    ("gdn write strength on the value only",
     "Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];",
     "Sh[(int64_t)i * dk + j] += (b * vh[i] - u[i]) * kh[j];"),
    ("gdn read-out before the rank-1 update",
     "    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];\n    for (int i = 0; i < dv; ++i) {\n      double acc = 0.0;\n      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * qh[j];\n      o[(int64_t)h * dv + i] = acc;\n    }\n",
     "    for (int i = 0; i < dv; ++i) {\n      double acc = 0.0;\n      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * qh[j];\n      o[(int64_t)h * dv + i] = acc;\n    }\n    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];\n"),
    ("gdn decay after the rank-1 update",
     "    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] *= a;\n    for (int i = 0; i < dv; ++i) {\n      double acc = 0.0;\n      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * kh[j];\n      u[i] = acc;\n    }\n    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];\n",
     "    for (int i = 0; i < dv; ++i) {\n      double acc = 0.0;\n      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * kh[j];\n      u[i] = acc;\n    }\n    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];\n    for (int i = 0; i < dv; ++i)\n      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] *= a;\n"),
    ("gdn read-out with the key",
     "for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * qh[j];",
     "for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * kh[j];"),
]


@pytest.mark.parametrize("name,orig,slip", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, orig, slip):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"the oracle source no longer holds the text this case mutates: {name}"
    mutated = tmp_path / "fmoe_oracle_mutated.c"
    mutated.write_text(src.replace(orig, slip))
    so = tmp_path / "liboracle_mutated.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                           "-std=c11", str(mutated), "-o", str(so), "-lm"])
    env = dict(os.environ, FMOE_ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"), "-q", "-x",
                        "-p", "no:cacheprovider", "-m", "not gpu"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"no pin failed with the planted mistake '{name}':\n{r.stdout[-2000:]}"
