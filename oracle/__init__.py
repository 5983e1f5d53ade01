"""The oracle: a plain CPU reference of the ALHR inference path. Test infrastructure only."""
