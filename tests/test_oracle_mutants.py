"""Plants plausible mistakes in copies of the oracle's C source and requires
every one of them to fail at least one pin (CPU only).

This is the evidence that the pins constrain the oracle: a dropped term, a
wrong sign or index, or a transposed operand anywhere in it is caught.
Each mutant is compiled into a temporary directory; the real oracle is not
touched.  Every mutation keeps all memory accesses in bounds (see MUTANTS).
"""
import pytest

import oracle
from pins import ALL_PINS

# Each mutant keeps every index in range (argued per line), so no mutant reads
# outside its arrays: key coordinates stay in [0, L) and bias indices in
# [0, 2k-2] because the window start stays inside [i' - (k-1), i'] or is
# clamped there.
MUTANTS = {
    # scores
    "drop_scale": [("dot * scale + bias", "dot + bias")],
    "scale_not_sqrt": [("const double scale = 1.0 / sqrt((double)D);", "const double scale = 1.0 / (double)D;")],
    "drop_bias": [("dot * scale + bias", "dot * scale")],
    "transpose_rpb": [("rpb[((size_t)h * nb + by[ty]) * nb + bx[tx]]",
                       "rpb[((size_t)h * nb + bx[tx]) * nb + by[ty]]")],
    # i' - s' is in [0, k-1], so the flipped index stays in [0, 2k-2]
    "bias_index_sign": [("bias_idx[t] = s + t - ip + k - 1;", "bias_idx[t] = ip - s - t + k - 1;")],
    "dot_wrong_operand": [("dot += qv[c] * kv[c];", "dot += qv[c] * qv[c];")],
    "dot_drops_last_channel": [("for (int c = 0; c < D; ++c) dot += qv[c] * kv[c];",
                                "for (int c = 0; c < D - 1; ++c) dot += qv[c] * kv[c];")],
    # window rule: start i' - k/3 differs from i' - k/2 for k >= 5 and keeps
    # the start within [i' - (k-1), i'] after the clamp
    "window_off_centre": [("int s = ip - r;", "int s = ip - k / 3;")],
    # g + s + t <= g + Lg - 1 <= L - 1
    "no_dilation_stride": [("keys[t] = g + d * (s + t);", "keys[t] = g + (s + t);")],
    # d * (ceil(L/d) - 1) <= L - 1, and i / d <= ceil(L/d) - 1
    "group_offset_dropped": [("int g = i % d;", "int g = 0;")],
    # softmax
    "softmax_exp_sign": [("sc[t] = exp(sc[t] - m);", "sc[t] = exp(m - sc[t]);"),
                         ("row[t] = exp(row[t] - m);", "row[t] = exp(m - row[t]);")],
    "softmax_not_normalised": [("const double pw = sc[ty * k + tx] / sum;", "const double pw = sc[ty * k + tx];"),
                               ("for (int t = 0; t < n; ++t) row[t] /= sum;", "")],
    # weighted sum: ky[tx] is still a row in [0, H), kx[ty] a column in [0, W)
    "av_transposed_gather": [("const double *vv = v + base + ((size_t)ky[ty] * W + kx[tx]) * D;",
                              "const double *vv = v + base + ((size_t)ky[tx] * W + kx[ty]) * D;"),
                             ("const double *vv = vs + ((size_t)ky[ty] * W + kx[tx]) * D;",
                              "const double *vv = vs + ((size_t)ky[tx] * W + kx[ty]) * D;")],
    "av_uses_keys": [("const double *vv = v + base +", "const double *vv = kk + base +")],
    # backward (every index unchanged, only the arithmetic)
    "bwd_drops_softmax_mean": [("const double ds = sc[n] * (dp[n] - pdp);", "const double ds = sc[n] * dp[n];")],
    "bwd_mean_unweighted": [("pdp += sc[ty * k + tx] * dot;", "pdp += dot;")],
    "bwd_dp_uses_query": [("dot += g[c] * vv[c];", "dot += g[c] * qv[c];")],
    "bwd_dq_unscaled": [("dqv[c] += ds * kk[key + c] * scale;", "dqv[c] += ds * kk[key + c];")],
    "bwd_dk_uses_key": [("dk[key + c] += ds * qv[c] * scale;", "dk[key + c] += ds * kk[key + c] * scale;")],
    "bwd_dv_uses_ds": [("dv[key + c] += sc[n] * g[c];", "dv[key + c] += ds * g[c];")],
    "bwd_drpb_transposed": [("drpb_acc[((size_t)h * nb + by[ty]) * nb + bx[tx]] += ds;",
                             "drpb_acc[((size_t)h * nb + bx[tx]) * nb + by[ty]] += ds;")],
    # dropout and its generator (indices unchanged)
    "philox_lo_hi_swapped": [("unsigned int n1 = (unsigned int)prod1;", "unsigned int n1 = (unsigned int)(prod1 >> 32);")],
    "philox_key_not_bumped": [("            k0 += 0x9E3779B9u;\n", "")],
    "dropout_not_rescaled": [("? 1.0 / (1.0 - p) : 0.0;", "? 1.0 : 0.0;")],
    "dropout_keeps_the_dropped": [("return w[e & 3] >= drop_threshold(p)", "return w[e & 3] < drop_threshold(p)")],
    "dropout_counter_not_grouped": [("unsigned long long blk = e >> 2;", "unsigned long long blk = e;")],
    "dropout_bwd_dv_unmasked": [("dv[key + c] += f[n] * sc[n] * g[c];", "dv[key + c] += sc[n] * g[c];")],
    "dropout_bwd_dp_unmasked": [("dp[ty * k + tx] = f[ty * k + tx] * dot;", "dp[ty * k + tx] = dot;")],
    "bwd_drpb_uses_p": [("drpb_acc[((size_t)h * nb + by[ty]) * nb + bx[tx]] += ds;",
                         "drpb_acc[((size_t)h * nb + by[ty]) * nb + bx[tx]] += sc[n];")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = oracle.SOURCE.read_text()
    for old, new in MUTANTS[name]:
        assert old in src, f"mutation site not found: {old!r}"
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(src)
    orc = oracle.Oracle(oracle.compile_c(c, tmp_path / "libmutant.so"))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
