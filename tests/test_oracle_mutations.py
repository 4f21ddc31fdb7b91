"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of oracle/ep_oracle.cpp (a
reversed loop, an off-by-one, a dropped term, a transposed index, a wrong
rounding), builds it, and runs the pin suite (tests/test_oracle_pins.py) against
that build.  The suite must fail for every mutant.  CPU only.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ep_oracle.cpp")

MUTANTS = {
    "receive order reversed": (
        "            for (int32_t t = 0; t < T; ++t) {\n"
        "                const int64_t g = (int64_t)s * T + t;\n"
        "                if (is_token_in_rank[g * R + d]) {\n"
        "                    send_head",
        "            for (int32_t t = T - 1; t >= 0; --t) {\n"
        "                const int64_t g = (int64_t)s * T + t;\n"
        "                if (is_token_in_rank[g * R + d]) {\n"
        "                    send_head"),
    "channel start off by one": (
        "return std::min<int64_t>(c * q, T);", "return std::min<int64_t>(c * q + (c > 0), T);"),
    "rank prefix drops last token": (
        "            for (int32_t t = 0; t < T; ++t)\n"
        "                running += is_token_in_rank[((int64_t)i * T + t) * R + d];",
        "            for (int32_t t = 0; t + 1 < T; ++t)\n"
        "                running += is_token_in_rank[((int64_t)i * T + t) * R + d];"),
    "combine drops bias1": (
        "acc[c] += bf16_bits_to_double(bias1[g * H + c]);",
        "acc[c] += 0.0 * bf16_bits_to_double(bias1[g * H + c]);"),
    "combine drops last rank": (
        "        for (int32_t d = 0; d < R; ++d) {\n"
        "            const int32_t h = send_head[g * R + d];\n"
        "            if (h < 0) continue;\n"
        "            const int64_t row = recv_rank_offset[d] + h;",
        "        for (int32_t d = 0; d < R - 1; ++d) {\n"
        "            const int32_t h = send_head[g * R + d];\n"
        "            if (h < 0) continue;\n"
        "            const int64_t row = recv_rank_offset[d] + h;"),
    "expert to rank transposed": ("in_row[e / L] = 1;", "in_row[e % R] = 1;"),
    "local id transposed": ("here ? e % L : -1;", "here ? e / L : -1;"),
    "rounding truncates": ("std::nearbyint(scaled)", "std::trunc(scaled)"),
    "recv channel prefix off by one": (
        "channel_prefix_matrix[((int64_t)s * R + d) * C + (c - 1)]",
        "channel_prefix_matrix[((int64_t)s * R + d) * C + c]"),
    "ll combine unweighted": (
        "acc[c] += w * bf16_bits_to_double(row[c]);", "acc[c] += bf16_bits_to_double(row[c]);"),
    "ll src_info stores the rank": (
        "src_info[list * cap + slot] = t;", "src_info[list * cap + slot] = s;"),
    "ll layout range shifted": ("const int64_t begin = slot;", "const int64_t begin = slot + (s > 0);"),
    "expert count per token": (
        "num_tokens_per_expert[(int64_t)s * E + e] += 1;", "num_tokens_per_expert[(int64_t)s * E + e] = 1;"),
    "fp8 scale uses the wrong range": (
        "amax > 0.0f ? 448.0f / amax : 0.0f", "amax > 0.0f ? 240.0f / amax : 0.0f"),
    "fp8 rounding truncates": (
        "double r = std::ldexp(std::nearbyint(std::ldexp(a, -qexp)), qexp);",
        "double r = std::ldexp(std::trunc(std::ldexp(a, -qexp)), qexp);"),
    "ll mask ignores the destination": (
        "(rank_mask[s] != 0 || rank_mask[d] != 0)", "(rank_mask[s] != 0)"),
    "lb reduce drops the original gradient": (
        "double acc = bf16_bits_to_double(expert_grads[(int64_t)e * W + c]);", "double acc = 0.0;"),
    "weights leak to other ranks": (
        "here ? topk_weights[g * K + k] : 0.0f;", "topk_weights[g * K + k];"),
    "fp32 combine in descending rank order": (
        "for (int32_t dst = 0; dst < R; ++dst) {          // ascending destination rank",
        "for (int32_t dst = R - 1; dst >= 0; --dst) {"),
    "fp32 combine accumulates in double": (
        "std::vector<float> sum32(H);", "std::vector<double> sum32(H);"),
    "fp32 combine adds bias1 before bias0": (
        "            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias0[g * H + c]);\n"
        "        if (bias1 != nullptr)\n"
        "            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias1[g * H + c]);",
        "            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias1[g * H + c]);\n"
        "        if (bias1 != nullptr)\n"
        "            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias0[g * H + c]);"),
    "fp32 combined weights skip the last rank": (
        "w32 = w32 + recv_topk_weights[(recv_rank_offset[dst] + h) * K + k];",
        "if (dst < R - 1) w32 = w32 + recv_topk_weights[(recv_rank_offset[dst] + h) * K + k];"),
    "fp32 ll combine in k order": ("std::sort(visit.begin(), visit.end());", ""),
    "fp32 ll combine rounds the product": (
        "chain[c] = std::fma(w32, bf16_bits_to_float(yrow[c]), chain[c]);",
        "chain[c] = w32 * bf16_bits_to_float(yrow[c]) + chain[c];"),
    "fp32 lb reduce in descending replica order": (
        "if (replicas.empty()) continue;                     // untouched",
        "if (replicas.empty()) continue; std::reverse(replicas.begin(), replicas.end());"),
    "fp32 lb reduce starts from zero": (
        "float g32 = bf16_bits_to_float(expert_grads[(int64_t)e * W + c]);", "float g32 = 0.0f;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    mutant = tmp_path / "mutant.cpp"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-fPIC", "-shared", "-ffp-contract=off",
                           str(mutant), "-o", str(lib)])
    env = dict(os.environ, EP_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch the planted mistake {name!r}:\n{r.stdout[-2000:]}"
