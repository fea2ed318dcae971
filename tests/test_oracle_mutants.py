"""The pins catch plausible mistakes: each case copies the oracle's C source,
plants one mistake (a dropped term, a wrong sign or index, a swapped
operand, a wrong widening), builds it and runs the pin tests against that
build, which must fail; the allocator cases do the same to a copy of the
oracle allocator and run the brute-force payload model on it, the caching
cases to a copy of the caching allocator under the prefix-cache pins, and
the quantizer cases to a copy of the E4M3 quantizer under its pin against
torch's cast.  (The mistakes live only in these temporary copies.)"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "oracle.c")

# name: (text in oracle.c, replacement)
MUTANTS = {
    "softmax scale dropped": ("x[t] = scale * acc;", "x[t] = acc;"),
    "kv head of a query head": ("        int g = h / G;\n        int64_t L = context_lens[s];\n        if (L <= 0) continue;\n"
                                "        if (L > (int64_t)max_blocks * block_size) { status = -1; continue; }\n"
                                "        const int32_t *bt = block_tables + (int64_t)s * max_blocks;\n        int bad = 0;",
                                "        int g = h % Hkv;\n        int64_t L = context_lens[s];\n        if (L <= 0) continue;\n"
                                "        if (L > (int64_t)max_blocks * block_size) { status = -1; continue; }\n"
                                "        const int32_t *bt = block_tables + (int64_t)s * max_blocks;\n        int bad = 0;"),
    "exponent sign": ("double w = exp(x[t] - mx);", "double w = exp(mx - x[t]);"),
    "slot offset": ("return (int64_t)bt[t / block_size] * block_size + t % block_size;",
                    "return (int64_t)bt[t / block_size] * block_size + (t + 1) % block_size;"),
    "K read for V": ("o[d] += w * pool_value(v_pool, vbase + d, kv_dtype, v_scale);",
                     "o[d] += w * pool_value(k_pool, vbase + d, kv_dtype, v_scale);"),
    "query elements reversed": ("acc += widen(q, qbase + d, q_dtype) * pool_value(k_pool, kbase + d, kv_dtype, k_scale);",
                                "acc += widen(q, qbase + (D - 1 - d), q_dtype) * pool_value(k_pool, kbase + d, kv_dtype, k_scale);"),
    "no normalisation": ("        for (int d = 0; d < D; ++d) o[d] /= den;\n        free(x);\n    }\n    return status;\n}\n\n/*\n * Causal",
                         "        free(x);\n    }\n    return status;\n}\n\n/*\n * Causal"),
    "bf16 widening": ("uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    "f16 widening": ("else v = ldexp((double)(m | 1024), e - 25);", "else v = ldexp((double)(m | 1024), e - 24);"),
    "e4m3 exponent bias": ("else v = ldexp((double)(8 + m), e - 10);", "else v = ldexp((double)(8 + m), e - 11);"),
    "causal limit": ("int64_t upto = L - n + (t - query_start[s]) + 1;", "int64_t upto = L - n + (t - query_start[s]);"),
    "FP8 V scaled by the K scale": ("o[d] += w * pool_value(v_pool, vbase + d, kv_dtype, v_scale);",
                                    "o[d] += w * pool_value(v_pool, vbase + d, kv_dtype, k_scale);"),
    "FP8 K scale dropped": ("acc += widen(q, qbase + d, q_dtype) * pool_value(k_pool, kbase + d, kv_dtype, k_scale);",
                            "acc += widen(q, qbase + d, q_dtype) * pool_value(k_pool, kbase + d, kv_dtype, 1.0);"),
    "chunk kv head of a query head": ("        int g = h / G;\n        const int32_t *bt = block_tables + (int64_t)s * max_blocks;",
                                      "        int g = h % Hkv;\n        const int32_t *bt = block_tables + (int64_t)s * max_blocks;"),
    "f16 subnormal exponent": ("if (e == 0) v = ldexp((double)m, -24);", "if (e == 0) v = ldexp((double)m, -25);"),
    "context length off by one": ("        int64_t L = context_lens[s];\n        if (L <= 0) continue;",
                                  "        int64_t L = context_lens[s] - 1;\n        if (L <= 0) continue;"),
}


def _build_and_run(d, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return "the planted mistake must replace exactly one place"
    tag = "m%d" % list(MUTANTS).index(name)
    mutant, lib = os.path.join(d, tag + ".c"), os.path.join(d, "liboracle_%s.so" % tag)
    open(mutant, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o",
                           lib, mutant, "-lm"])
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=dict(os.environ, ORACLE_LIBRARY=lib),
                       capture_output=True, text=True, timeout=600)
    if r.returncode == 0:
        return "no pin caught it"
    if "failed" not in r.stdout:
        return r.stdout[-2000:]
    return None


@pytest.fixture(scope="module")
def c_outcomes(tmp_path_factory):
    """Build each mutant oracle library and run the pins against it, the runs
    side by side (independent processes)."""
    from concurrent.futures import ThreadPoolExecutor
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    with ThreadPoolExecutor(max_workers=max(2, min(len(MUTANTS), os.cpu_count() or 2))) as ex:
        futures = {name: ex.submit(_build_and_run, d, name) for name in MUTANTS}
        return {name: f.result() for name, f in futures.items()}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_pins_catch_planted_mistake(name, c_outcomes):
    assert c_outcomes[name] is None, "%s: %s" % (name, c_outcomes[name])


# Planted mistakes in the Python allocator (class Allocator, the first class
# of oracle/allocator.py): (text, replacement, which occurrence).
ALLOC_MUTANTS = {
    "copy-on-write skipped": ("elif self.ref[bt[j]] > 1:", "elif False:", 0),
    "fork leaves refcounts": ("            self.ref[b] += 1\n        self.seqs[child]", "            pass\n        self.seqs[child]", 0),
    "freed blocks lost": ("self.free.append(b)", "pass", 0),
    "fresh block unreferenced": ("                self.ref[b] = 1\n                bt.append(b)",
                                 "                self.ref[b] = 0\n                bt.append(b)", 0),
    "block index of a token": ("j = t // bs", "j = (t + 1) // bs", 0),
    "freed blocks to the front": ("self.free.append(b)", "self.free.appendleft(b)", 0),
    "freed in reverse table order": ("        bt, _ = self.seqs.pop(sid)\n        for b in bt:",
                                     "        bt, _ = self.seqs.pop(sid)\n        for b in reversed(bt):", 0),
    "share without refcounts": ("        for b in blocks:\n            self.ref[b] += 1\n",
                                "        for b in blocks:\n            pass\n", 0),
    "copy pair reversed": ("pairs.append((bt[j], b))", "pairs.append((b, bt[j]))", 0),
    "copy keeps the old block's count": ("                self.ref[bt[j]] -= 1\n", "", 0),
    "fork child starts empty": ("        self.seqs[child] = [list(bt), n]", "        self.seqs[child] = [list(bt), 0]", 0),
    "failed append not rolled back": ("                if not self.free:\n                    self._restore(snap)\n",
                                      "                if not self.free:\n", 0),
    "failure not counted": ("                    self.alloc_failures += 1\n", "", 0),
    "copies not counted": ("                self.cow_copies += 1\n", "", 0),
    "slot in the table's first block": ("            slots.append(bt[j] * bs + t % bs)",
                                        "            slots.append(bt[0] * bs + t % bs)", 0),
}
# closed-form allocator pins tried when the brute-force model does not catch a mistake
ALLOC_PINS = ["test_worked_example_allocator_growth", "test_allocator_exhaustion_is_atomic",
              "test_fork_then_append_copies_partial_block_once_per_writer",
              "test_free_queue_takes_from_the_front_and_frees_to_the_back_in_table_order"]


def _mutant_allocator_module(old, new, which):
    import types
    src = open(os.path.join(ROOT, "oracle", "allocator.py")).read()
    at = -1
    for _ in range(which + 1):
        at = src.index(old, at + 1)
    src = src[:at] + new + src[at + len(old):]
    mod = types.ModuleType("oracle_allocator_mutant")
    exec(compile(src, "oracle_allocator_mutant", "exec"), mod.__dict__)
    return mod


def _mutant_allocator(old, new, which):
    return _mutant_allocator_module(old, new, which).Allocator


@pytest.mark.parametrize("name", list(ALLOC_MUTANTS))
def test_allocator_pins_catch_planted_mistake(name):
    import numpy as np
    import synth
    from test_oracle_pins import run_ops
    Broken = _mutant_allocator(*ALLOC_MUTANTS[name])
    caught = False
    for seed in range(3000):
        nb = 4 + seed % 3
        a = Broken(nb, 2, list(np.random.default_rng(seed).permutation(nb)))
        try:
            run_ops(a, synth.random_ops(seed, 8, max_seqs=4, max_append=4), 2)
        except (AssertionError, IndexError, KeyError, ValueError):
            caught = True
            break
    if not caught:              # counters and the free-queue order are pinned by closed-form cases
        import test_oracle_pins as pins
        saved = pins.Allocator
        pins.Allocator = Broken
        try:
            for pin in ALLOC_PINS:
                try:
                    getattr(pins, pin)()
                except (AssertionError, IndexError, KeyError, ValueError):
                    caught = True
        finally:
            pins.Allocator = saved
    assert caught, "no pin caught: %s" % name


# Planted mistakes in the caching allocator (class CachingAllocator of
# oracle/allocator.py), caught by the prefix-cache pins that do not involve
# the product: the prefix payload model, the closed-form hit counts, the
# eviction order and the all-or-nothing prompt registration.
CACHE_MUTANTS = {
    "evicts the newest released block": ("b = self.lru.pop(0)", "b = self.lru.pop()"),
    "released cached block goes back to the free queue": ("if b in self.key_of:\n                self.lru.append(b)",
                                                          "if False:\n                self.lru.append(b)"),
    "block key without its parent": ("key = (parent, tuple(block_toks))", "key = (self.ROOT, tuple(block_toks))"),
    "a hit takes no reference": ("            self.ref[b] += 1\n        n_cached", "            pass\n        n_cached"),
    "lookup skips a missed block": ("            if b is None:\n                break",
                                    "            if b is None:\n                continue"),
    "partial blocks registered": ("if t % bs == bs - 1:", "if True:"),
    "lookups counted in tokens": ("self.lookups += len(toks) // bs", "self.lookups += len(toks)"),
    "chain restarts after the cached blocks": ("        self.chain[sid] = node\n        st, slots, _",
                                               "        self.chain[sid] = self.ROOT\n        st, slots, _"),
    "revived block left in the LRU list": ("            if self.ref[b] == 0:\n                self.lru.remove(b)\n",
                                           "            pass\n"),
    "counters bumped by a refused prompt": (
        "        if st != OK:\n            self._restore(snap)\n            return st, 0, []\n        self.lookups",
        "        if st != OK:\n            self._restore(snap)\n            self.lookups += 1\n            return st, 0, []\n"
        "        self.lookups"),
    "evicted before the free queue is empty": ("        if self.free:\n            return self.free.popleft()\n",
                                               "        if self.free and not self.lru:\n            return self.free.popleft()\n"),
    "eviction keeps the key": ("            del self.cache[self.key_of.pop(b)]\n", "            self.key_of.pop(b)\n"),
    "released blocks at the front of the LRU list": ("            if b in self.key_of:\n                self.lru.append(b)",
                                                      "            if b in self.key_of:\n                self.lru.insert(0, b)"),
    "fork drops the token ids": ("            self.tokens[child] = None if t is None else list(t)\n",
                                 "            self.tokens[child] = None\n"),
}
CACHE_PINS = ["test_caching_oracle_payload_model", "test_hit_counts_closed_form",
              "test_freed_cached_blocks_are_evicted_oldest_first", "test_prompt_that_does_not_fit_changes_nothing",
              "test_forked_sequence_keeps_registering_its_blocks"]


@pytest.mark.parametrize("name", list(CACHE_MUTANTS))
def test_prefix_cache_pins_catch_planted_mistake(name, monkeypatch):
    import test_prefix_cache as pins
    old, new = CACHE_MUTANTS[name]
    monkeypatch.setattr(pins, "CachingAllocator", _mutant_allocator_module(old, new, 0).CachingAllocator)
    caught = []
    for pin in CACHE_PINS:
        try:
            getattr(pins, pin)()
        except (AssertionError, IndexError, KeyError, ValueError):
            caught.append(pin)
    assert caught, "no pin caught: %s" % name


# Planted mistakes in the oracle's E4M3 quantizer, caught by the pin against
# torch's float8_e4m3fn cast (exact ties included).
QUANT_MUTANTS = {
    "ties rounded away from zero": ("np.where(even_hi, hi, lo)", "hi"),
    "ties rounded toward zero": ("np.where(even_hi, hi, lo)", "lo"),
    "nearest taken the wrong way": ("dl < dh", "dl > dh"),
    "scale multiplied instead of divided": ("inv = np.float32(1.0) / np.float32(scale)", "inv = np.float32(scale)"),
    "sign dropped": ("code = np.where(np.signbit(y), code | 0x80, code).astype(np.uint8)",
                     "code = code.astype(np.uint8)"),
}


@pytest.mark.parametrize("name", list(QUANT_MUTANTS))
def test_quantizer_pins_catch_planted_mistake(name, monkeypatch):
    import inspect
    import textwrap

    import oracle
    import test_oracle_pins as pins
    old, new = QUANT_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(oracle.quantize_e4m3))
    assert src.count(old) == 1, "the planted mistake must replace exactly one place"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "quantize_e4m3_mutant", "exec"), ns)
    monkeypatch.setattr(oracle, "quantize_e4m3", ns["quantize_e4m3"])
    caught = False
    for scale in (1.0, 0.125, 0.37):
        try:
            pins.test_e4m3_quantize_matches_torch_cast_and_saturates(scale)
        except AssertionError:
            caught = True
            break
    assert caught, "no pin caught: %s" % name


# Planted mistakes in the oracle's Python helpers (oracle/__init__.py):
# (function, text, replacement, the pins expected to catch it).
PY_MUTANTS = {
    "append writes V into K": ("kv_append", "        k_pool[blk, :, off, :] = k_new[i]\n",
                               "        k_pool[blk, :, off, :] = v_new[i]\n",
                               ["test_worked_example_kv_append_lands_in_block_9"]),
    "append writes at negative slots": ("kv_append", "        if sl < 0:\n            continue\n", "",
                                        ["test_worked_example_kv_append_lands_in_block_9"]),
    "copy moves only K": ("block_copy", "    v_pool[dst] = vs\n", "", ["test_block_copy_copies_only_that_block"]),
    "FP8 append writes at negative slots": ("kv_append_fp8", "        if sl < 0:\n            continue\n", "",
                                            ["test_fp8_append_places_torch_codes_at_the_slots"]),
    "FP8 append puts V codes in the K pool": ("kv_append_fp8", "        k_codes[blk, :, off, :] = kq[i]\n",
                                              "        k_codes[blk, :, off, :] = vq[i]\n",
                                              ["test_fp8_append_places_torch_codes_at_the_slots"]),
    "FP8 K and V scales swapped": ("paged_attention_kv", "float(np.float32(k_scale)),\n        float(np.float32(v_scale))",
                                   "float(np.float32(v_scale)),\n        float(np.float32(k_scale))",
                                   ["test_fp8_attention_equals_attention_on_dequantized_values"]),
    "default scale 1/D": ("paged_attention", "        scale = 1.0 / math.sqrt(D)\n", "        scale = 1.0 / D\n",
                          ["test_two_token_closed_form_pins_scale_and_sign"]),
    "chunk default scale 1/D": ("paged_attention_chunk", "        scale = 1.0 / math.sqrt(D)\n",
                                "        scale = 1.0 / D\n", [("test_chunk_equals_sdpa_with_causal_mask",
                                                                  ("float32", 4, 4, 64, 16))]),
    "sampled items' row and head swapped": ("paged_attention",
                                            "    its_s = np.ascontiguousarray(its[:, 0])\n    its_h = np.ascontiguousarray(its[:, 1])\n",
                                            "    its_s = np.ascontiguousarray(its[:, 1])\n    its_h = np.ascontiguousarray(its[:, 0])\n",
                                            [("test_contiguous_equals_sdpa", ("float32", 4, 4, 64, 16, 35))]),
}


@pytest.mark.parametrize("name", list(PY_MUTANTS))
def test_python_helper_pins_catch_planted_mistake(name, monkeypatch):
    import inspect
    import textwrap

    import torch

    import oracle
    import test_oracle_pins as pins
    fn, old, new, pin_names = PY_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn)))
    assert src.count(old) == 1, "the planted mistake must replace exactly one place"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "oracle_helper_mutant", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    caught = False
    for pin in pin_names:
        pin, args = (pin, ()) if isinstance(pin, str) else pin
        args = tuple(getattr(torch, a) if isinstance(a, str) else a for a in args)
        try:
            getattr(pins, pin)(*args)
        except (AssertionError, IndexError, ValueError):
            caught = True
    assert caught, "no pin caught: %s" % name


def test_swapped_dtype_codes_are_caught(monkeypatch):
    """The oracle tells its C code the element type by a code; swapping the
    bf16 and f16 codes is caught by the exact-widening pin."""
    import torch

    import oracle
    import test_oracle_pins as pins
    monkeypatch.setitem(oracle._DT, torch.bfloat16, 2)
    monkeypatch.setitem(oracle._DT, torch.float16, 1)
    with pytest.raises(AssertionError):
        pins.test_narrow_types_widen_exactly(torch.bfloat16)
