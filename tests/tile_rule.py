"""The rule by which the library cuts segments into rows of its tile table.

The pages define only the grouping (the segmented gather of the Punica
README, "How?"): perm, indptr and the active list. How the SGMV kernels cut
each segment into units of work is a launch detail of this library, stated
in include/lora.h (lora_segments_t.tiles): every active segment, in order,
is cut into runs of at most t tokens, where t = lora_tile_tokens_for(T, n);
row = {adapter, first position in perm, token count, segment index}; the
rows after the last run are {-1, 0, 0, -1}. The tests derive the expected
table from the oracle's grouping with this rule and compare the library's
table with it bit for bit."""


def expected_tiles(indptr, active, n_active, t):
    rows = []
    for s in range(int(n_active)):
        a = int(active[s])
        first, end = int(indptr[a]), int(indptr[a + 1])
        for off in range(first, end, t):
            rows.append([a, off, min(t, end - off), s])
    return rows


def tile_tokens(T, n_adapters):
    """Tokens per tile row as include/lora.h states it: 4 for a decode-like
    batch (T <= 64 and T <= 2 * n_adapters), else 64."""
    return 4 if (T <= 64 and T <= 2 * n_adapters) else 64
