"""Host-side block manager oracle: the page pool of the PagedAttention pages.

Test infrastructure only.  The product has its own C++ block manager; this
plain Python model of the pages' simulation is what it is checked against.
Nothing in the product path imports this module.

Sources:
  "Atención paginada en modelos de lenguaje grandes (LLM)" (7minutos.es,
  a translation of a Marktechpost notebook article):
    - section 2 (PagePool, PagedRequest): the pool is a flat array of equal
      pages of 16 tokens with a free list and a per-page reference count; a
      page whose count drops to zero returns to the free list at once.  A
      request's block_table maps logical page i to a physical page id; a new
      physical page is claimed only when the token count crosses a page
      boundary.
    - section 3 (prefix sharing): share() raises a page's reference count
      without allocating; cow_copy() allocates a new page and lowers the
      original's count, and the other holders keep the original.
    - section 4 (utilisation): naive reservation of the maximum length versus
      ceil(tokens / 16) pages per request.
  "PagedAttention" (e-fortepiano.pl wiki mirror), "Descripció": blocks are
  reference-counted and copied on write at block granularity.

Readings where the pages are silent:
  - a fresh pool hands out the lowest free page id first (the worked example
    gets page 13 after pages 0..12 were taken);
  - a page is copied on write only while more than one block table holds it;
    the last holder writes in place;
  - a request's slot for logical position p is
    block_table[p // page_size] * page_size + p % page_size.
"""
from __future__ import annotations

import heapq
import math
from dataclasses import dataclass, field

PAGE_SIZE = 16


class PoolExhausted(RuntimeError):
    pass


class PagePool:
    """Flat array of equal-size physical pages with a free list and refcounts."""

    def __init__(self, num_pages: int, page_size: int = PAGE_SIZE):
        if num_pages <= 0 or page_size <= 0:
            raise ValueError("num_pages and page_size must be positive")
        self.num_pages = num_pages
        self.page_size = page_size
        self.refcount = [0] * num_pages
        self._free = list(range(num_pages))
        heapq.heapify(self._free)

    def num_free(self) -> int:
        return len(self._free)

    def allocate(self) -> int:
        if not self._free:
            raise PoolExhausted("no free page")
        page = heapq.heappop(self._free)
        self.refcount[page] = 1
        return page

    def share(self, page: int) -> None:
        self._check_live(page)
        self.refcount[page] += 1

    def free(self, page: int) -> None:
        self._check_live(page)
        self.refcount[page] -= 1
        if self.refcount[page] == 0:
            heapq.heappush(self._free, page)

    def cow_copy(self, page: int) -> int:
        """New private page for one holder of `page`; the original loses one reference."""
        self._check_live(page)
        new_page = self.allocate()
        self.refcount[page] -= 1
        return new_page

    def _check_live(self, page: int) -> None:
        if not (0 <= page < self.num_pages) or self.refcount[page] <= 0:
            raise ValueError(f"page {page} is not allocated")


@dataclass
class PagedRequest:
    """One inference request: a block table plus its token count."""

    pool: PagePool
    block_table: list = field(default_factory=list)
    num_tokens: int = 0

    def generate_token(self):
        """Account for one more token.

        Returns (slot, cow) where slot is the physical slot the token's K/V goes
        to and cow is a (src, dst) page pair when the tail page was shared and
        had to be copied first, else None.
        """
        ps = self.pool.page_size
        pos = self.num_tokens
        cow = None
        if pos % ps == 0:
            self.block_table.append(self.pool.allocate())
        else:
            tail = self.block_table[-1]
            if self.pool.refcount[tail] > 1:
                new_page = self.pool.cow_copy(tail)
                self.block_table[-1] = new_page
                cow = (tail, new_page)
        self.num_tokens += 1
        return slot_of(self.block_table, pos, ps), cow

    def share_prefix_of(self, other: "PagedRequest") -> None:
        """Point this (empty) request's block table at all of other's pages."""
        if self.block_table:
            raise ValueError("share_prefix_of needs an empty request")
        for page in other.block_table:
            self.pool.share(page)
        self.block_table = list(other.block_table)
        self.num_tokens = other.num_tokens

    def release(self) -> None:
        for page in self.block_table:
            self.pool.free(page)
        self.block_table = []
        self.num_tokens = 0


def slot_of(block_table, pos: int, page_size: int = PAGE_SIZE) -> int:
    return block_table[pos // page_size] * page_size + pos % page_size


def pages_needed(tokens: int, page_size: int = PAGE_SIZE) -> int:
    return math.ceil(tokens / page_size)


def kv_bytes_per_token(layers: int, heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V (factor 2) for every layer and head: the per-token KV cost."""
    return 2 * layers * heads * head_dim * elem_bytes


def naive_utilisation(token_counts, max_seq_len: int) -> float:
    """Tokens written over slots reserved when every request reserves max_seq_len."""
    return sum(token_counts) / (max_seq_len * len(token_counts))


def paged_utilisation(token_counts, page_size: int = PAGE_SIZE) -> float:
    """Tokens written over slots of the pages actually claimed."""
    pages = sum(pages_needed(t, page_size) for t in token_counts)
    return sum(token_counts) / (pages * page_size)
