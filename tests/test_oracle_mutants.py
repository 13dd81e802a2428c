"""Each planted mistake in a copy of the oracle must fail at least one pin.

The mistakes are the plausible ones: an off-by-one in a mask, the window read
as w+1 keys, a wrong GQA head map, a dropped scale, K and V swapped, a dropped
term in the log-sum-exp, ignored lengths or input_pos, a missing
normalisation, the wrong default decode scale.  Copies are built in a
temporary directory from ``oracle/oracle.c`` with one textual substitution
each; the real oracle is never modified.
"""
import pytest

import oracle
from oracle_pins import PINS

MUTANTS = {
    "causal_off_by_one": ("if (causal && j > pos) visible = 0;",
                          "if (causal && j >= pos) visible = 0;"),
    "window_w_plus_1": ("if (window > 0 && j <= pos - window) visible = 0;",
                        "if (window > 0 && j < pos - window) visible = 0;"),
    "gqa_modulo_map": ("const long hkv = hq / group;\n            const int k_len",
                       "const long hkv = hq % Hkv;\n            const int k_len"),
    "scale_dropped": ("score[j] = scale * dot + mask[j];", "score[j] = dot + mask[j];"),
    "k_v_swapped": ("dot += q[d] * Kb[j * D + d];\n                score[j] = scale * dot + mask[j];",
                    "dot += q[d] * Vb[j * D + d];\n                score[j] = scale * dot + mask[j];"),
    "decode_k_v_swapped": ("dot += q[d] * Kb[j * D + d];\n                score[j] = scale * dot;",
                           "dot += q[d] * Vb[j * D + d];\n                score[j] = scale * dot;"),
    "lse_missing_max": ("LSE[(b * Hq + hq) * (long)n_rows + r] = mx + log(l);",
                        "LSE[(b * Hq + hq) * (long)n_rows + r] = log(l);"),
    "q_lengths_ignored": ("int visible = (i < q_len) && (j < k_len);", "int visible = (j < k_len);"),
    "k_lengths_ignored": ("int visible = (i < q_len) && (j < k_len);", "int visible = (i < q_len);"),
    "input_pos_ignored": ("const long pos = (long)input_pos + i;\n    for (long j = 0; j < Sk; ++j) {",
                          "const long pos = i;\n    for (long j = 0; j < Sk; ++j) {"),
    "not_normalised": ("const double p = score[j] / l;\n                if (p == 0.0)",
                       "const double p = score[j];\n                if (p == 0.0)"),
    "decode_scale": ("const double scale = 1.0 / sqrt((double)D);", "const double scale = 1.0 / (double)D;"),
    "decode_lse_missing_max": ("if (LSE) LSE[b * Hq + hq] = mx + log(l);", "if (LSE) LSE[b * Hq + hq] = log(l);"),
    "decode_gqa_modulo": ("const long hkv = hq / group;\n            const int len",
                          "const long hkv = hq % Hkv;\n            const int len"),
    "page1_causal_strict": ("out[i * n_kv + j] = (j <= offset + i) ? 0.0 : -INFINITY;",
                            "out[i * n_kv + j] = (j < offset + i) ? 0.0 : -INFINITY;"),
    "page1_window_wide": ("const int visible = (j <= pos) && (j > pos - window_size);",
                          "const int visible = (j <= pos) && (j >= pos - window_size);"),
    "flex_softcap_inner": ("sj = softcap * tanh(sj / softcap);", "sj = softcap * tanh(sj);"),
    "flex_softcap_outer": ("sj = softcap * tanh(sj / softcap);", "sj = tanh(sj / softcap);"),
    "flex_scale_dropped": ("double sj = scale * dot;", "double sj = dot;"),
    "flex_alibi_sign": ("(q_pos - (double)j)", "((double)j - q_pos)"),
    "flex_alibi_kv_head": ("sj += alibi_slopes[hq]", "sj += alibi_slopes[kv_head]"),
    "flex_doc_ignored": ("if (doc_q[i] != doc_kv[j]) mask[j] = -INFINITY;", "if (0) mask[j] = -INFINITY;"),
    "flex_doc_kv_by_row": ("if (doc_q[i] != doc_kv[j]) mask[j] = -INFINITY;",
                           "if (doc_q[i] != doc_kv[i]) mask[j] = -INFINITY;"),
    "flex_gqa_modulo": ("const long kv_head = hq / group;", "const long kv_head = hq % Hkv;"),
    "flex_lse_missing_max": ("if (LSE) LSE[row_id] = mx + log(lsum);", "if (LSE) LSE[row_id] = log(lsum);"),
    "flex_not_normalised": ("const double pj = score[j] / lsum;", "const double pj = score[j];"),
    "paged_slot_by_block": ("const double *kr = K_cache + ((blk * block_size + j % block_size) * Hkv + kvh) * D;",
                            "const double *kr = K_cache + ((blk * block_size + j / block_size) * Hkv + kvh) * D;"),
    "paged_table_ignored": ("const long blk = block_tables[b * max_blocks + j / block_size];\n"
                            "                const double *kr",
                            "const long blk = b * max_blocks + j / block_size;\n"
                            "                const double *kr"),
    "paged_head_stride": ("const double *vr = V_cache + ((blk * block_size + j % block_size) * Hkv + kvh) * D;",
                          "const double *vr = V_cache + ((blk * block_size + j % block_size) + kvh) * D;"),
    "paged_v_from_k": ("const double *vr = V_cache +", "const double *vr = K_cache +"),
    "paged_scale": ("const double qk_scale = 1.0 / sqrt((double)D);", "const double qk_scale = 1.0 / (double)D;"),
    "paged_lse_missing_max": ("if (LSE) LSE[b * Hq + hq] = mx + log(den);",
                              "if (LSE) LSE[b * Hq + hq] = log(den);"),
    "rbs_centroid_sum": ("c[d] = acc / (j1 - j0);", "c[d] = acc / BS;"),
    "rbs_radius_squared": ("if (sqrt(ss) > rmax) rmax = sqrt(ss);", "if (ss > rmax) rmax = ss;"),
    "rbs_quantile_low": ("sorted_quantile(sorted, nkb, 0.5);", "sorted_quantile(sorted, nkb, 0.4);"),
    "rbs_beta_unclipped": ("bt = bt < 0.0 ? 0.0 : (bt > 1.0 ? 1.0 : bt);", "bt = bt;"),
    "rbs_degenerate_beta": ("bt = r > r_low ? 1.0 : 0.0;", "bt = 1.0;"),
    "rbs_rescue_no_norm": ("lr[i - i0] = (dot + sqrt(qq) * rb) * inv_sqrt_d;",
                           "lr[i - i0] = (dot + rb) * inv_sqrt_d;"),
    "rbs_scale": ("const double inv_sqrt_d = 1.0 / sqrt((double)D);", "const double inv_sqrt_d = 1.0 / (double)D;"),
    "rbs_lse_max_only": ("base[t * nkb + kb] = mb + log(sb);", "base[t * nkb + kb] = mb;"),
    "rbs_gqa_modulo": ("const long bh = b * Hkv + hq / group;", "const long bh = b * Hkv + hq % Hkv;"),
    "mask_alpha_inverted": ("(sb[k] >= mb + log(alpha_base))", "(sb[k] >= mb - log(alpha_base))"),
    "mask_band_wide": ("(qb - k < diagonal) && (k - qb < diagonal)", "(qb - k <= diagonal) && (k - qb <= diagonal)"),
    "mask_no_rescue": ("(sr[k] >= mr + log(alpha_rescue)) || band", "band"),
    "block_keep_ignored": ("if (!kr[j / 64]) mask[j] = -INFINITY;", "if (0) mask[j] = -INFINITY;"),
    "bwd_dq_scale": ("gq[d] += scale * ds * Kh[j * D + d];", "gq[d] += ds * Kh[j * D + d];"),
    "bwd_delta_zero": ("delta += prob[j] * dp;", "delta += 0.0 * dp;"),
    "bwd_unnormalised": ("prob[j] /= l;", "prob[j] /= 1.0;"),
    "bwd_dk_from_do": ("dKh[j * D + d] += scale * ds * q[d];", "dKh[j * D + d] += scale * ds * go[d];"),
    "bwd_dv_from_ds": ("dVh[j * D + d] += prob[j] * go[d];", "dVh[j * D + d] += ds * go[d];"),
    "bwd_one_head_per_group": ("for (long hq = hkv * group; hq < (hkv + 1) * group; ++hq)",
                               "for (long hq = hkv * group; hq < hkv * group + 1; ++hq)"),
    "visible_inverted": ("o[j] = (mask[j] == 0.0) ? 1 : 0;", "o[j] = (mask[j] == 0.0) ? 0 : 1;"),
    "visible_batch_stride": ("unsigned char *o = out + t * (long)Sk;",
                             "unsigned char *o = out + r * (long)Sk;"),
    "visible_window_dropped": ("mask_row(mask, i, Sk, causal, window, input_pos, k_len, q_len);\n"
                               "            unsigned char",
                               "mask_row(mask, i, Sk, causal, 0, input_pos, k_len, q_len);\n"
                               "            unsigned char"),
    "bwd_mask_ignored": ("mask_row(mrow, i, Sk, causal, window, input_pos, k_len, q_len);",
                         "mask_row(mrow, i, Sk, 0, 0, input_pos, Sk, Sq);"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique in oracle.c"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(old, new))
    lib = oracle.build(str(src), str(tmp_path / f"lib{name}.so"))
    mutant = oracle.Oracle(lib)
    failed = None
    for pin in PINS:  # one failing pin is enough; stop at the first
        try:
            pin(mutant)
        except AssertionError:
            failed = pin.__name__
            break
    assert failed, f"no pin catches the planted mistake {name}"
