"""The C ABI against the boundary the hot path was specified with.

The pages give no API; the boundary was fixed beforehand as a list of C entry
points (store, attention and its workspace size, block copy, debug status,
last error, and the host block manager). Every one of those names must be
declared in include/pa.h and exported by libpa.so with the same parameter
list, or with a parameter list recorded below together with the reason for
the difference. A change to either side that is not recorded here fails.
"""

import ctypes
import os
import re

import pytest

import paged_kv_cache_heads_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(not os.path.exists(P.library_path()), reason="libpa.so not built")

# Entry points of the specified boundary, with their parameter names in order.
SPECIFIED = {
    "pa_store_kv": ["k", "v", "slot_mapping", "num_tokens", "k_cache", "v_cache", "cache", "stream"],
    "pa_attention": ["q", "k_cache", "v_cache", "block_tables", "max_blocks_per_seq", "context_lens",
                     "query_start_loc", "num_seqs", "num_q_tokens", "num_q_heads", "max_query_len", "scale",
                     "cache", "out", "workspace", "workspace_bytes", "stream"],
    "pa_attention_workspace_size": ["num_seqs", "num_q_heads", "max_context_len", "cache"],
    "pa_copy_blocks": ["src_dst_pairs", "num_pairs", "k_cache", "v_cache", "cache", "stream"],
    "pa_get_debug_status": ["stream", "host_flag"],
    "pa_last_error": [],
    "pa_bm_create": ["num_blocks", "block_size", "shuffle_seed", "out"],
    "pa_bm_destroy": ["bm"],
    "pa_bm_add_seq": ["bm", "seq_id", "num_tokens"],
    "pa_bm_fork": ["bm", "parent", "child", "shared_tokens"],
    "pa_bm_append_tokens": ["bm", "seq_id", "n", "slots_out", "cow_pairs_out", "num_cow_out"],
    "pa_bm_free_seq": ["bm", "seq_id"],
    "pa_bm_block_table": ["bm", "seq_ids", "n", "max_blocks", "table_out", "ctx_lens_out"],
    "pa_bm_num_free": ["bm"],
    "pa_bm_refcount": ["bm", "block"],
}

# Parameter lists that differ from the specified ones, and why.
DEPARTURES = {
    "pa_attention": (
        ["q", "k_cache", "v_cache", "block_tables", "max_blocks_per_seq", "context_lens", "query_start_loc",
         "num_seqs", "num_q_tokens", "num_q_heads", "max_query_len", "max_context_len", "scale", "cache", "out",
         "workspace", "workspace_bytes", "stream"],
        "max_context_len: a host bound on the context lengths, which live on the device. It bounds the "
        "per-sequence range check without a device-to-host read, so the call never synchronises."),
    "pa_attention_workspace_size": (
        ["num_seqs", "num_q_heads", "max_query_len", "max_context_len", "cache"],
        "max_query_len: a decode-only batch (1) needs no prefill scratch; the same arguments as "
        "the pa_attention call it sizes."),
    "pa_bm_create": (
        ["num_blocks", "block_size", "initial_free_order", "out"],
        "the initial free-list order is passed in as a permutation instead of a seed: random numbers the "
        "method draws are inputs, so the library and the oracle need no shared generator."),
    "pa_bm_add_seq": (
        ["bm", "seq_id", "num_tokens", "slots_out"],
        "slots_out returns the slot of every token of the new sequence (the prompt's slot mapping); "
        "NULL keeps the specified behaviour."),
    "pa_bm_fork": (
        ["bm", "parent", "child", "num_tokens"],
        "renamed only (same meaning: the tokens shared with the parent; negative = all)."),
    "pa_bm_append_tokens": (
        ["bm", "seq_id", "n", "slots_out", "cow_pair_out", "num_cow_out"],
        "renamed only: at most one copy-on-write pair per call (the last block is the only one written)."),
}


def declared():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(pa_\w+)\s*\(([^;{]*?)\)\s*;", text):
        name, params = m.group(1), m.group(2).strip()
        if params in ("", "void"):
            out[name] = []
            continue
        names = []
        for p in params.split(","):
            ident = re.findall(r"[A-Za-z_]\w*", p.split("/*")[0])
            names.append(ident[-1])
        out[name] = names
    return out


def test_every_specified_entry_point_is_declared_and_exported():
    decl = declared()
    lib = ctypes.CDLL(P.library_path())
    for name in SPECIFIED:
        assert name in decl, name
        assert hasattr(lib, name), name
        assert name in P.exported_symbols(), name


@pytest.mark.parametrize("name", sorted(SPECIFIED))
def test_parameter_list_is_the_specified_one_or_a_recorded_departure(name):
    got = declared()[name]
    if name in DEPARTURES:
        want, reason = DEPARTURES[name]
        assert reason
        assert got == want, (name, got)
        assert got != SPECIFIED[name]
    else:
        assert got == SPECIFIED[name], (name, got)


def test_get_debug_status_rejects_null_without_a_gpu():
    with pytest.raises(P.PAError) as e:
        P.load_library()
        st = P.load_library().pa_get_debug_status(None, None)
        P._check(st)
    assert e.value.status == P.PA_ERR_INVALID_ARG
