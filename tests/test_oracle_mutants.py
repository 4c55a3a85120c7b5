"""Plant plausible mistakes in a copy of the oracle's C source and check
that the pins catch every one. The mistakes are planted in the oracle, on the
CPU; the real oracle is untouched."""
import os

import pytest

import oracle
import oracle_pins

# (name, text in atlas_oracle.c, replacement)
MUTANTS = [
    ("window_off_by_one", "if (win_off == NULL) return x / L;", "if (win_off == NULL) return (x + 1) / L;"),
    ("varlen_window_search", "if (win_off[mid] <= x) lo = mid; else hi = mid - 1;",
     "if (win_off[mid] < x) lo = mid; else hi = mid - 1;"),
    ("partial_cube_extent", "return (b + 1) * c <= E ? c : E - b * c;", "return c;"),
    ("global_sees_detail", "if (!q_detail && k_detail) return 0;", "if (!q_detail && k_detail) return 1;"),
    ("detail_misses_global", "return m->aligned ? global_aligned(m, m->cube_of[q], k - m->N) : 1;",
     "return m->aligned ? global_aligned(m, m->cube_of[q], k - m->N) : 0;"),
    ("aligned_sees_all", "return m->aligned ? global_aligned(m, m->cube_of[q], k - m->N) : 1;",
     "return 1;"),
    ("aligned_upper_bound_inclusive", "g * E < (a + e) * e_glob;", "g * E <= (a + e) * e_glob;"),
    ("aligned_ratio_inverted", "return a * e_glob <= g * E && g * E < (a + e) * e_glob;",
     "return a * E <= g * e_glob && g * e_glob < (a + e) * E;"),
    ("aligned_axis_mixup", "int64_t gt = g / (m->h * m->w), gh = (g / m->w) % m->h, gw = g % m->w;",
     "int64_t gt = g / (m->h * m->w), gh = (g / m->h) % m->w, gw = g % m->w;"),
    ("aligned_cube_coords", "int64_t bt = c / (nh * nw), bh = (c / nw) % nh, bw = c % nw;",
     "int64_t bt = c / (nh * nw), bh = (c / nh) % nw, bw = c % nw;"),
    ("rope_sign", "y[off + 2 * k] = x0 * c - x1 * s;", "y[off + 2 * k] = x0 * c + x1 * s;"),
    ("rope_freq_width", "pow(theta, -2.0 * (double)k / (double)d)", "pow(theta, -2.0 * (double)k / (double)(d + 2))"),
    ("rope_wrong_axis", "rope_segment(xr, yr, d_t + d_h, d_w, p_w, theta);", "rope_segment(xr, yr, d_t + d_h, d_w, p_h, theta);"),
    ("rope_scale_mixup", "double p_h = (double)((r / W) % H) * s_h;", "double p_h = (double)((r / W) % H) * s_w;"),
    ("rope_pair_layout", "double x0 = x[off + 2 * k], x1 = x[off + 2 * k + 1];", "double x0 = x[off + k], x1 = x[off + k + d / 2];"),
    ("cube_local_transposed", "int64_t local = ((t - bt * ct) * eh + (h - bh * ch)) * ew + (w - bw * cw);",
     "int64_t local = ((h - bh * ch) * et + (t - bt * ct)) * ew + (w - bw * cw);"),
    ("cube_order_transposed", "int64_t before = bt * ct * H * W + et * (bh * ch) * W + et * eh * (bw * cw);",
     "int64_t before = bw * cw * H * T + ew * (bh * ch) * T + ew * eh * (bt * ct);"),
    ("dropped_scale", "logit[n_allowed] = scale * dot;", "logit[n_allowed] = dot;"),
    ("lse_missing_max", "lse[i] = m + log(sum);", "lse[i] = log(sum);"),
    ("unorder_not_inverse", "memcpy(dst + r * row_bytes, src + j * row_bytes, (size_t)row_bytes);",
     "memcpy(dst + j * row_bytes, src + r * row_bytes, (size_t)row_bytes);"),
    ("bwd_lse_missing_max", "lse[i] = log(sum) + m;", "lse[i] = log(sum);"),
    ("bwd_drops_delta", "double ds = p * (dpo - delta[i]);", "double ds = p * dpo;"),
    ("bwd_dk_unscaled", "dkj[d] += scale * ds * q[i * D + d];", "dkj[d] += ds * q[i * D + d];"),
    ("bwd_dv_uses_ds", "dvj[d] += p * dout[i * D + d];", "dvj[d] += ds * dout[i * D + d];"),
    ("bwd_dq_wrong_key", "dqi[d] += scale * ds * k[key[a] * D + d];",
     "dqi[d] += scale * ds * q[key[a] * D + d];"),
    ("bwd_delta_unweighted", "dl += exp(logit[a] - lse[i]) * dp[a];", "dl += dp[a];"),
    ("dot_drops_last_channel", "for (int64_t d = 0; d < D; ++d) dot += qi[d] * kr[d];",
     "for (int64_t d = 0; d + 1 < D; ++d) dot += qi[d] * kr[d];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(src.replace(old, new))
    so = oracle.build(str(mutant_c), str(tmp_path / f"lib{name}.so"))
    orc = oracle.Oracle(oracle.load(so))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception:  # a crash or an error also counts as caught
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
