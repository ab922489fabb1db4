"""Row-chunk and tier rules of the host dispatch (a8), restated from the pages.

Test infrastructure (see the package docstring).
"""


def chunk_plan(rows, width):
    """Split ``rows`` into consecutive chunks of at most ``width`` rows.

    lm_head_fp8_rows.rs, ``lm_head_fp8_run``: ``done`` advances by
    ``min(rows - done, W8A8_MAX_ROWS)`` on the W8A8 branch and by 16-row
    chunks above 16 on the W8A16 branch; lm_head_q6k.rs, ``lm_head_q6k_run``:
    ``min(m - done, MAX_M)``.  Returns a list of (offset, count); empty for 0.
    """
    if rows < 0 or width <= 0:
        raise ValueError("rows must be >= 0 and width > 0")
    plan = []
    done = 0
    while done < rows:
        m = min(rows - done, width)
        plan.append((done, m))
        done += m
    return plan


def select_tier(m, widths, present):
    """Narrowest present tier that covers ``m`` rows, or None.

    w4a16_gemv_tiers.rs, ``select_tier``: ``None`` when ``m`` is 0 or no
    present tier is at least ``m`` wide; never a tier narrower than ``m`` nor
    one that is absent.  ``widths`` ascending, ``present`` parallel booleans.
    Returns the index into ``widths``.
    """
    if m == 0:
        return None
    for i, w in enumerate(widths):
        if w >= m and present[i]:
            return i
    return None
