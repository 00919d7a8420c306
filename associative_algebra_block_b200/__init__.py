"""libaal: associative-algebra block projections on B200 (placeholder)."""
