"""The oracle's pins must catch plausible mistakes.  Each case plants one
mistake in the oracle (a dropped factor, a wrong sign or index, a swapped
operand, an off-by-one, a wrong tie rule) in a child process and runs the
CPU pin suites there; at least one pin must fail.  A control run with no
mistake must pass."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_SUITES = ["tests/test_oracle_pins.py", "tests/test_quant_pins.py",
              "tests/test_window_pins.py", "tests/test_prefix_cache.py"]

A, Q, P, C = "oracle.attention", "oracle.quant", "oracle.kv_pool", "oracle.prefix_cache"
MISTAKES = {
    "scale 1/d": (A, "attention_two_pass", "1.0 / math.sqrt(d) if scale is None",
                  "1.0 / d if scale is None"),
    "GQA head h % Hkv": (A, "attention_two_pass", "kv_h = h // group", "kv_h = h % Hkv"),
    "causal off by one": (A, "attention_two_pass", "max_visible = kv_len - q_tokens + qt",
                          "max_visible = kv_len - q_tokens + qt - 1"),
    "K in place of V": (A, "attention_two_pass", "weights @ v[:, kv_h, :]",
                        "weights @ k[:, kv_h, :]"),
    "normalised by the max": (A, "attention_two_pass", "weights /= weights.sum()",
                              "weights /= weights.max()"),
    "online rescale sign": (A, "online_softmax_stats", "l * math.exp(m - m_new)",
                            "l * math.exp(m_new - m)"),
    "tiled rescale dropped": (A, "attention_tiled",
                              "correction = math.exp(m - m_new) if m != -math.inf else 0.0",
                              "correction = 1.0 if m != -math.inf else 0.0"),
    "combine weight without e^(m_p - M)": (
        A, "combine_partitions",
        "ls * np.exp(np.where(np.isfinite(ms), ms, 0.0) - safe_M)", "ls"),
    "window one short": (A, "visible_positions", "start = max(len(head), kv_len - window)",
                         "start = max(len(head), kv_len - window + 1)"),
    "int ties half up": (Q, "quantize_rows", "q = np.rint(x / scale[..., None])",
                         "q = np.floor(x / scale[..., None] + 0.5)"),
    "int limit + 1": (Q, "quantize_rows", "scale = np.abs(x).max(axis=-1) / limit",
                      "scale = np.abs(x).max(axis=-1) / (limit + 1)"),
    "E4M3 bias 8": (Q, "e4m3_values", "2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    "E4M3 ties to odd": (Q, "e4m3_round", "(hi % 2 == 0)", "(hi % 2 == 1)"),
    "E4M3 scale to 240": (Q, "quantize_rows_fp8", "scale = np.abs(x).max(axis=-1) / E4M3_MAX",
                          "scale = np.abs(x).max(axis=-1) / 240.0"),
    "copy-on-write of a private tail": (P, "KVPool.append", "self.refs[table[-1]] > 1:",
                                        "self.refs[table[-1]] >= 1:"),
    "copy-on-write keeps the old reference": (P, "KVPool.append", "self.refs[old] -= 1",
                                              "self.refs[old] -= 0"),
    "release frees a shared block": (P, "KVPool.release", "if self.refs[blk] == 0:",
                                     "if self.refs[blk] <= 1:"),
    "prefix key without revision": (C, "prefix_key",
                                    "return (scope, revision, tuple(tokens[:end]))",
                                    "return (scope, tuple(tokens[:end]))"),
    "prefix key without context": (C, "prefix_key", "tuple(tokens[:end])",
                                   "tuple(tokens[max(0, end - 16):end])"),
    "split partition sees one key fewer": (A, "partition_stats",
                                           "hi = min(stop, max_visible + 1)",
                                           "hi = min(stop, max_visible)"),
    "split partition not normalised": (A, "partition_stats",
                                       "o[qt, h] = (p @ v[start:hi, kv_h, :]) / l[qt, h]",
                                       "o[qt, h] = p @ v[start:hi, kv_h, :]"),
    "share_prefix one block short": (P, "KVPool.share_prefix",
                                     "[:math.ceil(prefix / self.block_size)]",
                                     "[:prefix // self.block_size]"),
    "preflight ignores the shared tail": (P, "KVPool.blocks_needed",
                                          "need += 1", "need += 0"),
    "waste counted from logical tokens": (P, "KVPool.snapshot",
                                          '"internal_waste_tokens": capacity - payload',
                                          '"internal_waste_tokens": capacity - logical'),
    "int8 scale kept in float64": (Q, "stored_rows", "s32 = scale.astype(np.float32)",
                                   "s32 = scale"),
    "int8 zero row scale 0.5": (Q, "quantize_rows", "scale = np.where(scale == 0.0, 1.0, scale)",
                                "scale = np.where(scale == 0.0, 0.5, scale)"),
    "E4M3 negative zero kept": (Q, "e4m3_round", "neg = (y.ravel() < 0) & (mag != 0)",
                                "neg = (y.ravel() < 0)"),
    "E4M3 subnormal exponent": (Q, "e4m3_values", "2.0 ** (1 - 7)", "2.0 ** (0 - 7)"),
    "tiled causal mask one late": (A, "attention_tiled", "np.arange(s0, s1) > max_visible",
                                   "np.arange(s0, s1) > max_visible + 1"),
    "split drops the tail partition": (A, "attention_split_kv",
                                       "parts = max(1, -(-kv_len // partition))",
                                       "parts = max(1, kv_len // partition)"),
    "fill takes the smallest sharer": (P, "KVPool.fills", "fill[blk] = max(fill[blk], min(",
                                       "fill[blk] = min(fill[blk] or self.block_size, min("),
    "prefix hit stops a block early": (C, "PrefixCache.hit_tokens",
                                       "(run + 1) * bs <= len(tokens)",
                                       "(run + 2) * bs <= len(tokens)"),
    "prefix cache last writer wins": (C, "PrefixCache.publish", "if key not in self.blocks:",
                                      "if True:"),
    "cached blocks not referenced": (C, "PrefixCache.create_cached",
                                     "pool.refs[blk] += 1", "pool.refs[blk] += 0"),
    "truncate keeps a dropped block": (P, "KVPool.truncate",
                                       "keep = math.ceil(length / self.block_size)",
                                       "keep = length // self.block_size + 1"),
    "truncate frees a shared block": (P, "KVPool.truncate", "if self.refs[blk] == 0:",
                                      "if self.refs[blk] <= 1:"),
}


# the pin suites that cover each oracle module (the control runs them all)
SUITES_FOR = {
    A: ["tests/test_oracle_pins.py", "tests/test_window_pins.py"],
    Q: ["tests/test_quant_pins.py"],
    P: ["tests/test_oracle_pins.py", "tests/test_prefix_cache.py"],
    C: ["tests/test_prefix_cache.py"],
}


def _run(mistake):
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests")]))
    env.pop("ORACLE_MUTATION", None)
    if mistake is not None:
        env["ORACLE_MUTATION"] = json.dumps(mistake)
    suites = PIN_SUITES if mistake is None else SUITES_FOR[mistake[0]]
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", "-p", "oracle_mutation",
           "-p", "no:cacheprovider", *suites]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_control_without_mistake_passes():
    r = _run(None)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_pins_catch_planted_mistake(name):
    r = _run(MISTAKES[name])
    # 1 = some test failed (the pin caught it); anything else is a broken harness
    assert r.returncode == 1, (name, r.returncode, r.stdout[-2000:], r.stderr[-2000:])
    assert "mutation site not unique" not in r.stdout + r.stderr
